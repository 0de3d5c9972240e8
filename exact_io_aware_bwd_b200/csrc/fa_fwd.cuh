// Forward pass of exact attention on sm_100a: one thread block per
// (batch, query head, 128-row query block).
//
// Method (pages: "FlashAttention" glossary, opening list and online-softmax
// paragraph; "flash attention io aware", sections "Flash Attention
// Algorithm" and "Online Softmax"): the query block stays on chip while the
// key/value blocks of its head stream through a shared-memory ring; each
// score block S_j = Q K_j^T lives only in tensor memory; a running row max m
// and row sum l are kept and the partial output is rescaled when the max
// grows; only O and one logsumexp per row are written back.  Queries are the
// outer loop and key/value blocks the inner one, as in the "Flash Attention"
// glossary of inferensys ("for each query block, iterate over key-value
// blocks"); the other order on the chipfoundry page reaches the same result.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r of the block and tensor
//              memory lane r.  Reads S_j, applies mask and scale, updates
//              (m, l), writes P_j (16-bit) back over S_j, rescales O when
//              needed, and finally normalises O, stores it (via TMA) and lse.
//   warp 4     TMA producer: Q once, then K_0, K_1, V_0, K_2, V_1, ... in the
//              order the MMA warp consumes them, through an NSLOT ring.
//   warp 5     MMA issuer (one thread): S_{j+1} = Q K_{j+1}^T into the other
//              score buffer while the softmax warps work on S_j, then
//              O += P_j V_j with P_j read from tensor memory.
//
// Tensor memory (512 columns x 128 lanes x 32 bit): score buffers at columns
// [0,128) and [128,256) (P_j aliases the first 64 columns of its buffer as
// packed 16-bit pairs), O at [256, 256 + d).
//
// Running max: the max used for the exponentials (m_ref) is only moved when
// a row's max exceeds it by more than 8 (in log2 units), so that O and l are
// rescaled rarely; P = 2^(s - m_ref) <= 2^8 stays well inside bf16/fp16 range.
// O and l always share the same m_ref, so O / l is exact (the reference point
// of a softmax is arbitrary).
#pragma once

#include "sm100.cuh"

namespace fa {

struct FwdParams {
  CUtensorMap tm_q;  // [B*Hq][N][d], box 64 x 128
  CUtensorMap tm_k;  // [B*Hkv][N][d]
  CUtensorMap tm_v;
  CUtensorMap tm_o;  // [B*Hq][N][d] (store)
  float* lse;        // [B*Hq][N]
  int N, Hq, Hkv, group, BH, n_qtiles, n_ktiles;
  float scale_log2;  // scale * log2(e)
};

template <int HD>
struct FwdLayout {
  static constexpr int kBoxBytes = 128 * 128;        // 128 rows x 64 columns x 2 B
  static constexpr int kChunks = HD / 64;            // 64-column boxes per tile
  static constexpr int kTileBytes = 128 * HD * 2;    // one 128-row tile
  static constexpr int kSlots = HD == 128 ? 6 : 8;   // K/V ring depth
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kTileBytes;
  static constexpr int kOffBar = kOffRing + kSlots * kTileBytes;
  // barriers: q_full, slot_full[kSlots], slot_empty[kSlots], s_full[2], p_full[2], pv_done, done
  static constexpr int kNumBars = 1 + 2 * kSlots + 2 + 2 + 1 + 1;
  static constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemPtr + 4;
  static constexpr int kSmemBytes = kOffAbort + 4;
  static constexpr int kDynSmem = kSmemBytes + 1024;  // slack for 1024-byte alignment
};

constexpr int kFwdThreads = 192;
constexpr uint32_t kKernFwd = 1;

template <int HD, bool BF16, bool CAUSAL>
__global__ void __launch_bounds__(kFwdThreads, 1) fa_fwd_kernel(const __grid_constant__ FwdParams p) {
  using L = FwdLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = sm + L::kOffQ;
  uint8_t* sRing = sm + L::kOffRing;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* slot_full = bars + 1;
  uint64_t* slot_empty = slot_full + L::kSlots;
  uint64_t* s_full = slot_empty + L::kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* done_bar = pv_done + 1;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sm + L::kOffTmemPtr);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kOffAbort);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // Work item, head-major: the blocks running at the same time mostly share
  // a head, so its K and V stay in L2; inside a head the largest query
  // blocks (the most key blocks under a causal mask) go first.
  const int item = blockIdx.x;
  const int bh = item / p.n_qtiles;
  const int qt = p.n_qtiles - 1 - item % p.n_qtiles;
  const int h = bh % p.Hq;
  const int b = bh / p.Hq;
  const int kvh = b * p.Hkv + h / p.group;
  const int n_kv = CAUSAL ? min(qt + 1, p.n_ktiles) : p.n_ktiles;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < L::kSlots; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    mbar_init(pv_done, 1);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_ptr, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const uint32_t tm_S0 = tmem;        // score buffer 0, columns [0, 128)
  const uint32_t tm_O = tmem + 256;   // output accumulator

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&p.tm_q);
      prefetch_tensormap(&p.tm_k);
      prefetch_tensormap(&p.tm_v);
      mbar_expect_tx(q_full, L::kTileBytes);
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_3d(sQ + c * L::kBoxBytes, &p.tm_q, q_full, c * 64, qt * 128, bh);
      int t = 0;
      auto load = [&](const CUtensorMap* map, int tile) -> bool {
        const int s = t % L::kSlots;
        if (t >= L::kSlots &&
            !mbar_wait(&slot_empty[s], ((t / L::kSlots) - 1) & 1, abort_flag, kKernFwd, 4, 0))
          return false;
        mbar_expect_tx(&slot_full[s], L::kTileBytes);
        uint8_t* dst = sRing + s * L::kTileBytes;
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(dst + c * L::kBoxBytes, map, &slot_full[s], c * 64, tile * 128, kvh);
        ++t;
        return true;
      };
      // consumption order of the MMA warp: K0, then (K_{j+1}, V_j) for each j
      bool ok = load(&p.tm_k, 0);
      for (int j = 0; ok && j < n_kv; ++j) {
        if (j + 1 < n_kv) ok = load(&p.tm_k, j + 1);
        if (ok) ok = load(&p.tm_v, j);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_f16(BF16, 128, 128, false, false);
      constexpr uint32_t kIdPV = idesc_f16(BF16, 128, HD, false, true);
      int t = 0;
      bool ok = mbar_wait(q_full, 0, abort_flag, kKernFwd, 5, 0);
      auto take = [&](int& slot) -> bool {
        slot = t % L::kSlots;
        if (!mbar_wait(&slot_full[slot], (t / L::kSlots) & 1, abort_flag, kKernFwd, 5, 1))
          return false;
        tc_fence_after();
        ++t;
        return true;
      };
      auto issue_s = [&](int j, int slot) {
        const uint32_t kb = smem_u32(sRing + slot * L::kTileBytes);
        const uint32_t qb = smem_u32(sQ);
        const uint32_t d_tm = tm_S0 + (j & 1) * 128;
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (k >> 2) * L::kBoxBytes + (k & 3) * 32;
          umma_ss(d_tm, sdesc_sw128(qb + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), kIdS,
                  k > 0);
        }
        umma_commit(&s_full[j & 1]);
        umma_commit(&slot_empty[slot]);
      };
      int slot = 0;
      if (ok && n_kv > 0) {
        ok = take(slot);
        if (ok) issue_s(0, slot);
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        if (j + 1 < n_kv) {
          // buffer (j+1)&1 still holds P_{j-1} until PV_{j-1} has completed
          if (j >= 1) ok = mbar_wait(pv_done, (j - 1) & 1, abort_flag, kKernFwd, 5, 2);
          if (ok) ok = take(slot);
          if (!ok) break;
          issue_s(j + 1, slot);
        }
        if (!mbar_wait(&p_full[j & 1], (j >> 1) & 1, abort_flag, kKernFwd, 5, 3)) break;
        tc_fence_after();
        if (!take(slot)) break;
        const uint32_t vb = smem_u32(sRing + slot * L::kTileBytes);
        const uint32_t p_tm = tm_S0 + (j & 1) * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_ts(tm_O, p_tm + k * 8, sdesc_sw128(vb + k * 2048, L::kBoxBytes, 1024), kIdPV,
                  (j > 0 || k > 0) ? 1u : 0u);
        umma_commit(&slot_empty[slot]);
        umma_commit(pv_done);
      }
      // Everything issued has completed once done_bar flips (also on abort).
      umma_commit(done_bar);
      mbar_wait(done_bar, 0, abort_flag, kKernFwd, 5, 4);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int r = tid;  // query row within the block == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int q_row = qt * 128 + r;
    const float c_log2 = p.scale_log2;
    float m_ref = -INFINITY;  // in log2 units of the scaled scores
    float l_sum = 0.f;
    bool ok = true;
    // Waits are made warp-uniform: tcgen05.ld/st are warp-collective, so a
    // warp either goes on together or leaves together (on abort).
    for (int j = 0; j < n_kv; ++j) {
      const int buf = j & 1;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&s_full[buf], (j >> 1) & 1, abort_flag, kKernFwd, 0, 0))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s[128];
      const uint32_t s_tm = tm_S0 + buf * 128 + lane_off;
      tmem_ld32(s_tm + 0, s);
      tmem_ld32(s_tm + 32, s + 32);
      tmem_ld32(s_tm + 64, s + 64);
      tmem_ld32(s_tm + 96, s + 96);
      tmem_ld_wait();
      // mask: keys past the end of the sequence, and keys after the query
      // inside the diagonal block of a causal problem
      const int kv0 = j * 128;
      const bool diag = CAUSAL && (j == qt);
      if (diag || kv0 + 128 > p.N) {
        const int lim = min(diag ? r : 127, p.N - 1 - kv0);  // last visible column
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > lim) s[c] = __float_as_uint(-INFINITY);
      }
      // row max with four independent chains (shorter dependency)
      float mx4[4] = {__uint_as_float(s[0]), __uint_as_float(s[1]), __uint_as_float(s[2]),
                      __uint_as_float(s[3])};
#pragma unroll
      for (int c = 4; c < 128; ++c) mx4[c & 3] = fmaxf(mx4[c & 3], __uint_as_float(s[c]));
      const float m_new = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * c_log2;
      if (j == 0) {
        m_ref = m_new;
      } else if (__any_sync(0xffffffffu, m_new > m_ref + 8.0f)) {
        // Move the reference max of every row of this warp (tcgen05.ld/st
        // are warp-wide), rescaling O and l; O is stable once PV_{j-1} is done.
        if (!__all_sync(0xffffffffu,
                        mbar_wait(pv_done, (j - 1) & 1, abort_flag, kKernFwd, 0, 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float m_upd = fmaxf(m_ref, m_new);
        const float corr = ex2_approx(m_ref - m_upd);
        m_ref = m_upd;
        l_sum *= corr;
#pragma unroll
        for (int c = 0; c < HD; c += 32) {
          uint32_t o[32];
          tmem_ld32(tm_O + lane_off + c, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
          tmem_st32(tm_O + lane_off + c, o);
        }
      }
      const float neg_m = -m_ref;
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(s[half * 64 + 2 * i]), c_log2, neg_m));
          const float p1 =
              ex2_approx(fmaf(__uint_as_float(s[half * 64 + 2 * i + 1]), c_log2, neg_m));
          ls4[i & 3] += p0 + p1;
          pk[i] = pack2<BF16>(p0, p1);
        }
        tmem_st32(tm_S0 + buf * 128 + lane_off + half * 32, pk);
      }
      l_sum += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[buf]);
    }
    // epilogue: O / l -> 16-bit, staged in the (now idle) Q tile, TMA store
    bool ep_ok = ok && n_kv > 0;
    if (ep_ok) ep_ok = mbar_wait(pv_done, (n_kv - 1) & 1, abort_flag, kKernFwd, 0, 2);
    ep_ok = __all_sync(0xffffffffu, ep_ok);
    if (ep_ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l_sum;
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        uint32_t o[32];
        tmem_ld32(tm_O + lane_off + c, o);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv_l,
                              __uint_as_float(o[2 * i + 1]) * inv_l);
        // columns c..c+31 = 4 chunks of 16 B in box c/64, logical chunk (c%64)/8 + u
        uint8_t* row_base = sQ + (c / 64) * L::kBoxBytes + r * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int chunk = ((c % 64) / 8 + u) ^ (r & 7);
          *reinterpret_cast<uint4*>(row_base + chunk * 16) =
              make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
      if (q_row < p.N)
        p.lse[static_cast<size_t>(bh) * p.N + q_row] = (m_ref + __log2f(l_sum)) * 0.69314718055994531f;
      fence_proxy_async_smem();
    }
    // every softmax thread reaches this barrier, whatever happened above
    named_barrier_sync(1, 128);
    if (tid == 0 && !*abort_flag) {
      for (int c = 0; c < L::kChunks; ++c)
        tma_store_3d(&p.tm_o, sQ + c * L::kBoxBytes, c * 64, qt * 128, bh);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
