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
// and writes its unnormalised O with the row max m and sum l (base 2); a
// second kernel merges the splits: m* = max m_s, l* = sum l_s 2^(m_s - m*),
// O = sum O_s 2^(m_s - m*) / l*, lse = ln 2 (m* + log2 l*).
//
// Inside a block (128 threads) pages are staged in shared memory by bulk
// copies (cp.async.bulk, the copy engine; completion counted in bytes on an
// mbarrier) into a ring of kStages page slots, so that several pages are in
// flight while one is used: warp 0 issues a page's copies (one per K row,
// into rows padded by 16 bytes so that one thread per key reads its row
// without bank conflicts, and one for the whole V page) and refills a slot
// as soon as every thread is done with it.  Scores take all 128 threads
// (128 / P threads per key, combined by shuffles), the softmax update one
// warp per row, and P V one thread per output column.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace fa {

constexpr uint32_t kKernDecode = 10;
constexpr uint32_t kKernDecodeMerge = 11;
constexpr uint32_t kStatusBadInput = 7;  // a block-table entry or sequence length out of range
constexpr int kDecodeThreads = 128;
constexpr int kDecodeMaxRows = 32;
constexpr int kDecodeMaxPage = 128;

struct DecodeParams {
  const void* q;          // [B][Hq][Nq][d]
  const void* kc;         // [num_pages][Hkv][P][d]
  const void* vc;
  const int* table;       // [B][max_pages]
  const int* lens;        // [B]
  float* part_o;          // [B][Hq][Nq][S][d]   unnormalised partial outputs
  float* part_ml;         // [B][Hq][Nq][S][2]   (m, l) in base 2
  void* o;                // [B][Hq][Nq][d]
  float* lse;             // [B][Hq][Nq]
  int B, Hq, Hkv, Nq, P, max_pages, num_pages, S, pages_per_split;
  float scale_log2;
};

// Page slots of the ring for page size P and row bound RB: as many as fit
// in about 100 KB (two blocks per SM), at least 2 and at most 8.
template <int HD>
__host__ __device__ inline int decode_stages(int P, int rb) {
  const int slot = P * (HD * 2 + 16) + P * HD * 2;
  const int fixed = rb * HD * 4 + rb * P * 4 + 3 * kDecodeMaxRows * 4 + 8 * 8;
  int st = (100 * 1024 - fixed) / slot;
  return st < 2 ? 2 : (st > 8 ? 8 : st);
}

// Splits of each (sequence, kv head): enough blocks for four full waves of
// two blocks per SM of a full B200, at least 4 pages a split.
__host__ __device__ inline int decode_splits(int B, int Hkv, int max_pages) {
  const int bh = B * Hkv > 0 ? B * Hkv : 1;
  int want = (4 * 2 * 148 + bh - 1) / bh;
  const int cap = max_pages / 4 > 1 ? max_pages / 4 : 1;
  want = want > cap ? cap : want;
  return want < 1 ? 1 : want;
}

inline size_t decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int d, int max_pages) {
  const int64_t S = decode_splits(B, Hkv, max_pages);
  const int64_t rows = static_cast<int64_t>(B) * Hq * Nq * S;
  return static_cast<size_t>(rows) * 4u * static_cast<size_t>(d + 2);
}

// Shared memory for page size P, row bound RB and the ring's slots (bytes,
// all offsets multiples of 16): the slots' K (padded rows) and V pages,
// fp32 queries [RB][HD], fp32 scores [RB][P], row state, slot barriers.
// Sized by RB and P so that two blocks fit on an SM.
template <int HD>
struct DecodeLayout {
  static constexpr int kKRow = HD * 2 + 16;  // padded K row, bytes
  int P, stages, off_k, off_v, off_q, off_s, off_row, off_bar, bytes;
  __host__ __device__ DecodeLayout(int page, int rb) : P(page) {
    stages = decode_stages<HD>(page, rb);
    const int kbuf = page * kKRow, vbuf = page * HD * 2;
    off_k = 0;                                   // K slots
    off_v = stages * kbuf;                       // V slots
    off_q = off_v + stages * vbuf;
    off_s = off_q + rb * HD * 4;
    off_row = off_s + rb * page * 4;
    off_bar = off_row + 3 * kDecodeMaxRows * 4;
    bytes = off_bar + 8 * 8;
  }
};

// RB: compile-time bound on the rows (4, 8, 16 or 32, the smallest >= R), so
// the per-row loops unroll to the rows that exist.
template <int HD, bool BF16, int RB>
__global__ void __launch_bounds__(kDecodeThreads) fa_decode_split_kernel(const __grid_constant__ DecodeParams p) {
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  const DecodeLayout<HD> lay(p.P, RB);
  constexpr int kKRow = DecodeLayout<HD>::kKRow;
  extern __shared__ __align__(16) uint8_t smem[];
  float* sQ = reinterpret_cast<float*>(smem + lay.off_q);
  float* sS = reinterpret_cast<float*>(smem + lay.off_s);
  float* sM = reinterpret_cast<float*>(smem + lay.off_row);
  float* sL = sM + kDecodeMaxRows;
  float* sC = sL + kDecodeMaxRows;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.off_bar);  // [stages]
  __shared__ int abort_flag;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.Hq / p.Hkv, R = G * p.Nq, P = p.P, NS = lay.stages;
  const int Lb = p.lens[b];
  const bool len_ok = Lb >= p.Nq && Lb <= p.max_pages * P;
  if (!len_ok && split == 0 && g == 0 && tid == 0) record_error(kStatusBadInput, kKernDecode, 0, 0);
  const int n_pages = len_ok ? (Lb + P - 1) / P : 0;
  const int pg0 = split * p.pages_per_split;
  const int pg1 = min(n_pages, pg0 + p.pages_per_split);

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&full[i], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  // queries of the block's rows (row r: head g*G + r / Nq, token r % Nq),
  // fp32 and scaled by scale * log2(e)
  for (int i = tid; i < R * HD; i += kDecodeThreads) {
    const int r = i / HD, c = i % HD;
    const int h = g * G + r / p.Nq, t = r % p.Nq;
    const T* qr = reinterpret_cast<const T*>(p.q) + ((static_cast<size_t>(b) * p.Hq + h) * p.Nq + t) * HD;
    sQ[i] = static_cast<float>(qr[c]) * p.scale_log2;
  }
  if (tid < kDecodeMaxRows) {
    sM[tid] = -INFINITY;
    sL[tid] = 0.f;
  }
  float acc[RB];  // thread c < HD: output column c of every row
#pragma unroll
  for (int r = 0; r < RB; ++r) acc[r] = 0.f;
  __syncthreads();

  // page pg -> slot (pg - pg0) % NS; a bad page id is recorded and its keys
  // treated as hidden: nothing is read for it and the slot's barrier is
  // completed by a plain arrival.  Issued by warp 0.
  auto page_id = [&](int pg) { return p.table[static_cast<size_t>(b) * p.max_pages + pg]; };
  auto issue = [&](int pg) {
    const int phys = page_id(pg);
    const int slot = (pg - pg0) % NS;
    uint64_t* bar = &full[slot];
    const bool good = phys >= 0 && phys < p.num_pages;
    if (lane == 0) {
      if (good)
        mbar_expect_tx(bar, static_cast<uint32_t>(2 * P * HD * 2));
      else
        mbar_arrive(bar);
    }
    __syncwarp();
    if (!good) return;
    uint8_t* sKb = smem + lay.off_k + slot * P * kKRow;
    uint8_t* sVb = smem + lay.off_v + slot * P * HD * 2;
    const size_t base = (static_cast<size_t>(phys) * p.Hkv + g) * P * HD;
    const uint8_t* kg = reinterpret_cast<const uint8_t*>(reinterpret_cast<const T*>(p.kc) + base);
    const uint8_t* vg = reinterpret_cast<const uint8_t*>(reinterpret_cast<const T*>(p.vc) + base);
    for (int j = lane; j < P; j += 32) bulk_load(sKb + j * kKRow, kg + static_cast<size_t>(j) * HD * 2, HD * 2, bar);
    if (lane == 0) bulk_load(sVb, vg, static_cast<uint32_t>(P * HD * 2), bar);
  };
  int issued = pg0;  // pages whose copies warp 0 has issued: [pg0, issued)
  if (warp == 0)
    for (; issued < pg1 && issued < pg0 + NS; ++issued) issue(issued);
  int consumed = pg0;  // pages fully used: [pg0, consumed); consumed <= issued
  for (int pg = pg0; pg < pg1; ++pg) {
    const int slot = (pg - pg0) % NS;
    const bool ok = mbar_wait(&full[slot], ((pg - pg0) / NS) & 1, &abort_flag, kKernDecode, 0, 1);
    if (__syncthreads_or(!ok)) break;
    const int phys = page_id(pg);
    const bool page_ok = phys >= 0 && phys < p.num_pages;
    if (!page_ok && tid == 0) record_error(kStatusBadInput, kKernDecode, 1, 0);
    const uint8_t* sK = smem + lay.off_k + slot * P * kKRow;
    const T* sV = reinterpret_cast<const T*>(smem + lay.off_v + slot * P * HD * 2);
    // scores: tpk = 128 / P threads per key, each over d / tpk features,
    // summed across the key's threads by shuffles; s[r][j] = q_r . k_j (log2
    // units), -inf where hidden (after the query, past the sequence, or a
    // bad page)
    {
      const int tpk = kDecodeThreads / P;          // 1, 2, 4 or 8 (P = 128 .. 16)
      const int j = tid / tpk, part = tid % tpk;   // the threads of a key are adjacent lanes
      const int n8 = HD / 8 / tpk;                 // 16-byte chunks per thread
      const int key = pg * P + j;
      float s[RB];
#pragma unroll
      for (int r = 0; r < RB; ++r) s[r] = 0.f;
      const uint8_t* kr = sK + j * kKRow;
      for (int c = 0; c < n8; ++c) {
        const int c8 = part * n8 + c;
        const uint4 kv = *reinterpret_cast<const uint4*>(kr + c8 * 16);
        const T* k8 = reinterpret_cast<const T*>(&kv);
        float kf[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) kf[e] = static_cast<float>(k8[e]);
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          if (r < R) {
            const float4 qa = *reinterpret_cast<const float4*>(sQ + r * HD + c8 * 8);
            const float4 qb = *reinterpret_cast<const float4*>(sQ + r * HD + c8 * 8 + 4);
            s[r] = fmaf(qa.x, kf[0], fmaf(qa.y, kf[1], fmaf(qa.z, kf[2], fmaf(qa.w, kf[3],
                   fmaf(qb.x, kf[4], fmaf(qb.y, kf[5], fmaf(qb.z, kf[6], fmaf(qb.w, kf[7], s[r]))))))));
          }
        }
      }
      for (int off = 1; off < tpk; off <<= 1) {
#pragma unroll
        for (int r = 0; r < RB; ++r) s[r] += __shfl_xor_sync(0xffffffffu, s[r], off);
      }
      if (part == 0) {
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          if (r < R) {
            const int t = r % p.Nq;
            const bool vis = page_ok && key <= Lb - p.Nq + t;
            sS[r * P + j] = vis ? s[r] : -INFINITY;
          }
        }
      }
    }
    __syncthreads();
    // online softmax update, one warp per row: new max, rescale factor, P
    for (int r = warp; r < R; r += kDecodeThreads / 32) {
      float* sr = sS + r * P;
      float mx = -INFINITY;
      for (int j = lane; j < P; j += 32) mx = fmaxf(mx, sr[j]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = sM[r];
      const float m_new = fmaxf(m_old, mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;  // no visible key yet: P = 0
      float sum = 0.f;
      for (int j = lane; j < P; j += 32) {
        const float e = ex2_approx(sr[j] - m_use);
        sr[j] = e;
        sum += e;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      __syncwarp();
      if (lane == 0) {
        const float corr = m_new == -INFINITY ? 1.f : ex2_approx(m_old - m_new);
        sC[r] = corr;
        sL[r] = sL[r] * corr + sum;
        sM[r] = m_new;
      }
    }
    __syncthreads();
    // O += P V, one thread per output column
    if (tid < HD) {
#pragma unroll
      for (int r = 0; r < RB; ++r)
        if (r < R) acc[r] *= sC[r];
      for (int j = 0; j < P; j += 4) {
        const float v0 = static_cast<float>(sV[(j + 0) * HD + tid]);
        const float v1 = static_cast<float>(sV[(j + 1) * HD + tid]);
        const float v2 = static_cast<float>(sV[(j + 2) * HD + tid]);
        const float v3 = static_cast<float>(sV[(j + 3) * HD + tid]);
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          if (r < R) {
            const float4 pr = *reinterpret_cast<const float4*>(sS + r * P + j);
            acc[r] = fmaf(pr.x, v0, fmaf(pr.y, v1, fmaf(pr.z, v2, fmaf(pr.w, v3, acc[r]))));
          }
        }
      }
    }
    __syncthreads();  // every thread is done with this slot and the scores
    consumed = pg + 1;
    if (warp == 0 && issued < pg1) issue(issued++);
  }
  // after an abort, copies still in flight land before the block exits:
  // warp 0 waits (bounded) for every page it issued and no one consumed.
  // pg0 <= consumed <= issued <= pg1 here (an empty split has all four
  // equal), so every slot index below is in [0, NS).
  if (warp == 0 && lane == 0)
    for (int pg = consumed; pg < issued; ++pg)
      mbar_wait_drain(&full[(pg - pg0) % NS], ((pg - pg0) / NS) & 1, kKernDecode, 0, 2);

  // partial results of this split: unnormalised O, (m, l)
  if (tid < HD) {
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      if (r < R) {
        const int h = g * G + r / p.Nq, t = r % p.Nq;
        const size_t row = ((static_cast<size_t>(b) * p.Hq + h) * p.Nq + t) * p.S + split;
        p.part_o[row * HD + tid] = acc[r];
      }
    }
  }
  if (tid < R) {
    const int h = g * G + tid / p.Nq, t = tid % p.Nq;
    const size_t row = ((static_cast<size_t>(b) * p.Hq + h) * p.Nq + t) * p.S + split;
    p.part_ml[row * 2 + 0] = sM[tid];
    p.part_ml[row * 2 + 1] = sL[tid];
  }
}

// Merge of the splits of one (sequence, query head, token): one block of HD
// threads, thread c owns output column c.
template <int HD, bool BF16>
__global__ void __launch_bounds__(HD) fa_decode_merge_kernel(const __grid_constant__ DecodeParams p) {
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  const size_t row = blockIdx.x;  // (b * Hq + h) * Nq + t
  const int c = threadIdx.x;
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
