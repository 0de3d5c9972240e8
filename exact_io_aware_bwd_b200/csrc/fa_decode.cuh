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
// Inside a block (128 threads) pages are staged in shared memory by
// asynchronous 16-byte copies (cp.async), double-buffered so that the next
// page is in flight while the current one is used; K rows are padded by 16
// bytes so that one thread per key reads its row without bank conflicts.
// Scores take all 128 threads (128 / P threads per key, combined by
// shuffles), the softmax update one warp per row, and P V one thread per
// output column.
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

__host__ __device__ inline int decode_splits(int B, int Hkv, int max_pages) {
  // enough blocks for two per SM of a full B200, never more than the pages
  const int want = (2 * 148 + B * Hkv - 1) / (B * Hkv > 0 ? B * Hkv : 1);
  return want < 1 ? 1 : (want > max_pages ? (max_pages > 0 ? max_pages : 1) : want);
}

inline size_t decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int d, int max_pages) {
  const int64_t S = decode_splits(B, Hkv, max_pages);
  const int64_t rows = static_cast<int64_t>(B) * Hq * Nq * S;
  return static_cast<size_t>(rows) * 4u * static_cast<size_t>(d + 2);
}

// Shared memory for page size P and row bound RB (bytes, all offsets
// multiples of 16): two page buffers (K padded, V), fp32 queries [RB][HD],
// fp32 scores [RB][P], row state.  Sized by RB so that more blocks fit on an
// SM when there are few rows.
template <int HD>
struct DecodeLayout {
  static constexpr int kKRow = HD * 2 + 16;  // padded K row, bytes
  int P, off_k, off_v, off_q, off_s, off_row, bytes;
  __host__ __device__ DecodeLayout(int page, int rb) : P(page) {
    const int kbuf = page * kKRow, vbuf = page * HD * 2;
    off_k = 0;                                   // K buffers 0, 1
    off_v = 2 * kbuf;                            // V buffers 0, 1
    off_q = off_v + 2 * vbuf;
    off_s = off_q + rb * HD * 4;
    off_row = off_s + rb * page * 4;
    bytes = off_row + 3 * kDecodeMaxRows * 4;
  }
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.Hq / p.Hkv, R = G * p.Nq, P = p.P;
  const int Lb = p.lens[b];
  const bool len_ok = Lb >= p.Nq && Lb <= p.max_pages * P;
  if (!len_ok && split == 0 && g == 0 && tid == 0) record_error(kStatusBadInput, kKernDecode, 0, 0);
  const int n_pages = len_ok ? (Lb + P - 1) / P : 0;
  const int pg0 = split * p.pages_per_split;
  const int pg1 = min(n_pages, pg0 + p.pages_per_split);

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

  // page pg -> buffer (pg - pg0) & 1; a bad page id is recorded and its
  // keys treated as hidden (nothing is read for it)
  auto page_id = [&](int pg) { return p.table[static_cast<size_t>(b) * p.max_pages + pg]; };
  auto issue = [&](int pg) {
    const int phys = page_id(pg);
    if (phys < 0 || phys >= p.num_pages) return;
    const int buf = (pg - pg0) & 1;
    uint8_t* sKb = smem + lay.off_k + buf * P * kKRow;
    uint8_t* sVb = smem + lay.off_v + buf * P * HD * 2;
    const size_t base = (static_cast<size_t>(phys) * p.Hkv + g) * P * HD;
    const uint8_t* kg = reinterpret_cast<const uint8_t*>(reinterpret_cast<const T*>(p.kc) + base);
    const uint8_t* vg = reinterpret_cast<const uint8_t*>(reinterpret_cast<const T*>(p.vc) + base);
    constexpr int kVecRow = HD / 8;  // 16-byte vectors per row
    for (int i = tid; i < P * kVecRow; i += kDecodeThreads) {
      const int j = i / kVecRow, c = i % kVecRow;
      cp_async16(sKb + j * kKRow + c * 16, kg + static_cast<size_t>(i) * 16);
      cp_async16(sVb + static_cast<size_t>(i) * 16, vg + static_cast<size_t>(i) * 16);
    }
  };
  if (pg0 < pg1) issue(pg0);
  cp_async_commit();
  for (int pg = pg0; pg < pg1; ++pg) {
    // the next page's copies go out before this page is used
    if (pg + 1 < pg1) issue(pg + 1);
    cp_async_commit();
    cp_async_wait<1>();  // every group but the newest has landed
    __syncthreads();
    const int phys = page_id(pg);
    const bool page_ok = phys >= 0 && phys < p.num_pages;
    if (!page_ok && tid == 0) record_error(kStatusBadInput, kKernDecode, 1, 0);
    const int buf = (pg - pg0) & 1;
    const uint8_t* sK = smem + lay.off_k + buf * P * kKRow;
    const T* sV = reinterpret_cast<const T*>(smem + lay.off_v + buf * P * HD * 2);
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
    __syncthreads();  // this buffer and the scores are rewritten next
  }
  cp_async_wait<0>();

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
