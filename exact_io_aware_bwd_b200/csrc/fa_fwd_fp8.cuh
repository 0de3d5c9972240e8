// FP8 forward pass of exact attention on sm_100a: Q, K and V as 8-bit E4M3
// codes with one dequantisation factor per tensor, O written in bf16 or fp16
// and one logsumexp per row, as in the 16-bit forward.
//
// Method: the FlashAttention-3 paragraph of the "FlashAttention" glossary
// and section "Flash Attention 2 and 3" of "flash attention io aware" name
// FP8 low-precision tensor cores for attention and give no further rule.
// The plainest reading, kept here: both products run on FP8 operands with
// fp32 accumulation, scores S = delta_q delta_k Q8 K8^T, probabilities P
// rounded to E4M3 for the second product, O = delta_v (P V8) / l, with the
// running max and sum of the online softmax exactly as in the 16-bit
// forward ("flash attention io aware", section "Online Softmax").
//
// Structure (the 16-bit forward's, with 8-bit operand tiles): one thread block
// per (batch, query head, pair of 128-row query blocks), or per couple of
// such pairs (n-1-c, c) of a head run back to back while a head has at most
// 64 pairs (equal work per block under a causal mask; the second pair's Q
// load and first products overlap the first pair's tail), 320 threads:
//   warps 0-3 / 4-7  softmax of query block 0 / 1 (thread r owns row r and
//              tensor-memory lane r); P goes to E4M3, four keys per 32-bit
//              tensor-memory column, over the first 32 columns of S_t.
//   warp 8     MMA issuer (tcgen05.mma kind::f8f6f4, one elected lane).
//   warp 9     TMA producer.
// A 128-row tile of d = 128 one-byte elements is one 128-byte-swizzled TMA
// box of 16 KB, so one K-major atom row holds a whole row of Q or K: the
// score product takes four MMAs of K = 32 (32 bytes each, the same byte step
// as the 16-bit kernels' K = 16).  V stays in its [key][d] layout and is read
// MN-major (d contiguous), which tcgen05 accepts for E4M3 operands: each MMA
// of the P V product covers 32 keys = four 8-row core groups, 4 KB of the tile.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,384),
// O1 [384,512).  The output tile is staged in its own 32 KB per block (the
// 16 KB query tile is too small for a 16-bit 128 x 128 tile).
#pragma once

#include "sm100.cuh"

namespace fa {

struct Fp8FwdParams {
  CUtensorMap tm_q;  // [B*Hq][N][128] E4M3 codes, box 128 x 128
  CUtensorMap tm_k;  // [B*Hkv][N][128]
  CUtensorMap tm_v;
  CUtensorMap tm_o;  // [B*Hq][N][128] 16-bit (store), box 64 x 128
  float* lse;        // [B*Hq][N]
  int N, Hq, Hkv, group, BH, n_pairs, n_ktiles;
  int fold;          // 1: a block runs query pairs n-1-c and c; 0: one pair
  float scale_log2;  // scale * delta_q * delta_k * log2(e)
  float delta_v;
};

struct Fp8FwdLayout {
  static constexpr int kTileBytes = 128 * 128;      // 128 rows x 128 one-byte elements
  static constexpr int kOutBoxBytes = 128 * 128;    // 128 rows x 64 16-bit columns
  static constexpr int kOutBytes = 2 * kOutBoxBytes;
  static constexpr int kSlots = 8;                  // K/V ring depth
  static constexpr int kOffQ = 0;                   // two query tiles
  static constexpr int kOffRing = 2 * kTileBytes;
  static constexpr int kOffOut = kOffRing + kSlots * kTileBytes;  // two output tiles
  static constexpr int kOffBar = kOffOut + 2 * kOutBytes;
  // barriers: q_full, slot_full[kSlots], slot_empty[kSlots], s_full[2], p_full[2], pv_done[2], done,
  // q_free
  static constexpr int kNumBars = 1 + 2 * kSlots + 6 + 1 + 1;
  static constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemPtr + 4;
  static constexpr int kSmemBytes = kOffAbort + 4;
  static constexpr int kDynSmem = kSmemBytes + 1024;  // slack for 1024-byte alignment
  static_assert(kDynSmem <= 232448, "shared memory budget");
};

constexpr int kFwdFp8Threads = 320;
constexpr uint32_t kKernFwdFp8 = 12;

// Instruction descriptor of tcgen05.mma kind::f8f6f4 with E4M3 A and B and an
// fp32 accumulator: D format F32 (bits 4-5 = 1), A/B format E4M3 (bits 7-9,
// 10-12 = 0), A/B major (bit 15 / 16: 0 K-major, 1 MN-major), N >> 3 (bits
// 17-22), M >> 4 (bits 24-28).
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Warp-wide kind::f8f6f4 MMAs (the whole converged warp calls, one elected
// lane issues): A and B from shared memory, or A from tensor memory.
__device__ __forceinline__ void umma8_ss_w(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ void umma8_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

// Four fp32 values -> four E4M3 codes in one 32-bit word, x0 in the low
// byte (round to nearest even, saturating to +-448).  cvt...e4m3x2 puts its
// first source in the upper byte of the 16-bit result.
__device__ __forceinline__ uint32_t pack4_e4m3(float x0, float x1, float x2, float x3) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(x0), "f"(x1), "f"(x2), "f"(x3));
  return r;
}

template <bool OUT_BF16, bool CAUSAL>
__global__ void __launch_bounds__(kFwdFp8Threads, 1) fa_fwd_fp8_kernel(const __grid_constant__ Fp8FwdParams p) {
  using L = Fp8FwdLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = sm + L::kOffQ;
  uint8_t* sRing = sm + L::kOffRing;
  uint8_t* sOut = sm + L::kOffOut;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* slot_full = bars + 1;
  uint64_t* slot_empty = slot_full + L::kSlots;
  uint64_t* s_full = slot_empty + L::kSlots;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* done_bar = pv_done + 2;
  uint64_t* q_free = done_bar + 1;  // every S product of a pair (the readers of sQ) has completed
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sm + L::kOffTmemPtr);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kOffAbort);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // head-major work order, query pairs with the most key blocks first; with
  // folding, pairs n-1-c and c of a head back to back
  const int n_couples = p.fold ? (p.n_pairs + 1) / 2 : p.n_pairs;
  const int bh = blockIdx.x / n_couples;
  const int cpl = blockIdx.x % n_couples;
  const int n_items = (!p.fold || p.n_pairs - 1 - cpl == cpl) ? 1 : 2;
  auto item_pair = [&](int it) { return it == 0 ? p.n_pairs - 1 - cpl : cpl; };
  const int h = bh % p.Hq;
  const int b = bh / p.Hq;
  const int kvh = b * p.Hkv + h / p.group;
  auto n_kv_of = [&](int pair, int t) {
    return CAUSAL ? min(2 * pair + 1 + t, p.n_ktiles) : p.n_ktiles;
  };

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    for (int s = 0; s < L::kSlots; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_ptr, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;

  if (warp == 9) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&p.tm_q);
      prefetch_tensormap(&p.tm_k);
      prefetch_tensormap(&p.tm_v);
      int n = 0;  // K/V tiles loaded (ring position), over both pairs
      auto load = [&](const CUtensorMap* map, int tile) -> bool {
        const int s = n % L::kSlots;
        if (n >= L::kSlots &&
            !mbar_wait(&slot_empty[s], ((n / L::kSlots) - 1) & 1, abort_flag, kKernFwdFp8, 9, 0))
          return false;
        mbar_expect_tx(&slot_full[s], L::kTileBytes);
        tma_load_3d(sRing + s * L::kTileBytes, map, &slot_full[s], 0, tile * 128, kvh);
        ++n;
        return true;
      };
      bool ok = true;
      for (int it = 0; ok && it < n_items; ++it) {
        const int pair = item_pair(it);
        // Q0, Q1 of the pair once the previous pair's S products (the last
        // readers of sQ) have completed
        if (it > 0) ok = mbar_wait(q_free, (it - 1) & 1, abort_flag, kKernFwdFp8, 9, 1);
        if (!ok) break;
        mbar_expect_tx(q_full, 2 * L::kTileBytes);
        for (int t = 0; t < 2; ++t)
          tma_load_3d(sQ + t * L::kTileBytes, &p.tm_q, q_full, 0, (2 * pair + t) * 128, bh);
        for (int j = 0; ok && j < n_kv_of(pair, 1); ++j) {
          ok = load(&p.tm_k, j);
          if (ok) ok = load(&p.tm_v, j);
        }
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdS = idesc_e4m3(128, 128, false, false);
    constexpr uint32_t kIdPV = idesc_e4m3(128, 128, false, true);
    const uint64_t dQ_k = sdesc_sw128(smem_u32(sQ), 16, 1024);     // Q tile 0, K-major
    const uint64_t dR_k = sdesc_sw128(smem_u32(sRing), 16, 1024);  // ring slot 0, K-major
    // ring slot 0 read MN-major: one 128-byte atom spans all d = 128 columns,
    // so the leading (MN) offset is never used; 8-key core groups are 1 KB apart
    const uint64_t dR_mn = sdesc_sw128(smem_u32(sRing), L::kTileBytes, 1024);
    auto wait_all = [&](uint64_t* bar, uint32_t parity, uint32_t site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, kKernFwdFp8, 8, site));
    };
    int n = 0;
    bool ok = true;
    auto take = [&](int& slot) -> bool {
      slot = n % L::kSlots;
      if (!wait_all(&slot_full[slot], (n / L::kSlots) & 1, 1)) return false;
      tc_fence_after();
      ++n;
      return true;
    };
    // Same staggered order as the 16-bit forward: S0_0 S1_0 PV0_0 | S0_1
    // PV1_0 S1_1 PV0_1 | ...; MMAs of this warp run in issue order, so S_t,j+1
    // may follow O_t += P_t,j V_j (which reads P over S_t) without a wait.
    auto issue_s = [&](int t, int kslot) {
      const uint32_t qo = t * L::kTileBytes, ko = kslot * L::kTileBytes;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma8_ss_w(tmem + t * 128, sdesc_add(dQ_k, qo + k * 32), sdesc_add(dR_k, ko + k * 32), kIdS,
                   k > 0);
      umma_commit_w(&s_full[t]);
    };
    // g: the tile's index over both pairs (barrier phase), j: its index in the pair
    auto issue_pv = [&](int t, int g, int j, int vslot) -> bool {
      if (!wait_all(&p_full[t], g & 1, 3)) return false;
      tc_fence_after();
      const uint32_t vo = vslot * L::kTileBytes;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma8_ts_w(tmem + 256 + t * 128, tmem + t * 128 + k * 8, sdesc_add(dR_mn, vo + k * 4096), kIdPV,
                   (j > 0 || k > 0) ? 1u : 0u);
      umma_commit_w(&pv_done[t]);
      return true;
    };
    int g0 = 0, g1 = 0;  // tiles of query block 0 / 1 in the pairs before this one
    for (int it = 0; ok && it < n_items; ++it) {
      const int pair = item_pair(it);
      const int n_kv0 = n_kv_of(pair, 0), n_kv1 = n_kv_of(pair, 1);
      if (!(ok = wait_all(q_full, it & 1, 0))) break;
      tc_fence_after();
      int kslot = 0, vslot = 0;
      if (!(ok = take(kslot))) break;
      if (n_kv0 > 0) issue_s(0, kslot);
      issue_s(1, kslot);
      umma_commit_w(&slot_empty[kslot]);
      if (n_kv1 == 1) umma_commit_w(q_free);  // the pair's last S
      if (!(ok = take(vslot))) break;
      if (n_kv0 > 0 && !(ok = issue_pv(0, g0, 0, vslot))) break;
      for (int j = 0; ok && j < n_kv1; ++j) {
        const bool next1 = j + 1 < n_kv1, next0 = j + 1 < n_kv0;
        if (next1 && !(ok = take(kslot))) break;
        if (next0) issue_s(0, kslot);
        if (!(ok = issue_pv(1, g1 + j, j, vslot))) break;
        umma_commit_w(&slot_empty[vslot]);  // V_j: read by both PV_j
        if (next1) {
          issue_s(1, kslot);
          umma_commit_w(&slot_empty[kslot]);  // K_j+1: read by both S_j+1
          if (j + 2 == n_kv1) umma_commit_w(q_free);  // the pair's last S
          if (!(ok = take(vslot))) break;
        }
        if (next0 && !(ok = issue_pv(0, g0 + j + 1, j + 1, vslot))) break;
      }
      g0 += n_kv0;
      g1 += n_kv1;
    }
    // every MMA this warp issued completes before tensor memory is freed
    umma_commit_w(done_bar);
    mbar_wait_drain(done_bar, 0, kKernFwdFp8, 8, 4);
  } else {
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;                 // query block of this warpgroup
    const int r = tid & 127;                 // row within the block == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tm_S = tmem + t * 128 + lane_off;
    const uint32_t tm_O = tmem + 256 + t * 128 + lane_off;
    const float c_log2 = p.scale_log2;
    const uint64_t c2 = f2pack(c_log2, c_log2);
    uint8_t* sOt = sOut + t * L::kOutBytes;
    int gt = 0;  // tiles of this query block in the pairs before this one
    bool ok = true;
    for (int it = 0; ok && it < n_items; ++it) {
    const int pair = item_pair(it);
    const int qtile = 2 * pair + t;
    const int q_row = qtile * 128 + r;
    const int n_kv = n_kv_of(pair, t);
    float m_ref = -INFINITY;  // in log2 units of the scaled scores
    float l_sum = 0.f;
    for (int j = 0; j < n_kv; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[t], (gt + j) & 1, abort_flag, kKernFwdFp8, t, 0))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32(tm_S + 0, s);
      tmem_ld32(tm_S + 32, s + 32);
      tmem_ld32(tm_S + 64, s + 64);
      tmem_ld32(tm_S + 96, s + 96);
      tmem_ld_wait();
      // keys past the end of the sequence, and keys after the query inside
      // the diagonal block of a causal problem
      const int kv0 = j * 128;
      const bool diag = CAUSAL && (j == qtile);
      if (diag || kv0 + 128 > p.N) {
        const int lim = min(diag ? r : 127, p.N - 1 - kv0);  // last visible column
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > lim) s[c] = __float_as_uint(-INFINITY);
      }
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(s[i]);
#pragma unroll
      for (int c = 8; c < 128; ++c) mx[c & 7] = fmaxf(mx[c & 7], __uint_as_float(s[c]));
#pragma unroll
      for (int i = 0; i < 4; ++i) mx[i] = fmaxf(mx[i], mx[i + 4]);
      const float m_new = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c_log2;
      if (j == 0) {
        m_ref = m_new;
      } else if (__any_sync(0xffffffffu, m_new > m_ref + 8.0f)) {
        // move the reference max of every row of this warp once
        // O_t += P_t,j-1 V_j-1 is done, rescaling O and l
        if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[t], (gt + j - 1) & 1, abort_flag, kKernFwdFp8, t, 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float m_upd = fmaxf(m_ref, m_new);
        const float corr = m_upd == -INFINITY ? 1.f : ex2_approx(m_ref - m_upd);
        const uint64_t corr2 = f2pack(corr, corr);
        m_ref = m_upd;
        l_sum *= corr;
#pragma unroll 1
        for (int c = 0; c < 128; c += 16) {
          uint32_t o[16];
          tmem_ld16(tm_O + c, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const uint64_t v = mul2(f2pack(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), corr2);
            o[i] = __float_as_uint(f2lo(v));
            o[i + 1] = __float_as_uint(f2hi(v));
          }
          tmem_st16(tm_O + c, o);
        }
      }
      // P = 2^(s c - m_ref) <= 2^8, to E4M3 over the first 32 columns of S
      // (four keys per column); l sums the fp32 values
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
      const uint64_t nm2 = f2pack(-m_use, -m_use);
      uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c = q4 * 32 + 4 * i;
          const uint64_t x01 = fma2(f2pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), c2, nm2);
          const uint64_t x23 = fma2(f2pack(__uint_as_float(s[c + 2]), __uint_as_float(s[c + 3])), c2, nm2);
          const uint64_t p01 = f2pack(ex2_approx(f2lo(x01)), ex2_approx(f2hi(x01)));
          const uint64_t p23 = f2pack(ex2_approx(f2lo(x23)), ex2_approx(f2hi(x23)));
          acc[(2 * i) & 3] = add2(acc[(2 * i) & 3], p01);
          acc[(2 * i + 1) & 3] = add2(acc[(2 * i + 1) & 3], p23);
          pk[i] = pack4_e4m3(f2lo(p01), f2hi(p01), f2lo(p23), f2hi(p23));
        }
        tmem_st8(tm_S + q4 * 8, pk);
      }
      const uint64_t a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
      const uint64_t a = add2(a01, a23);
      l_sum += f2lo(a) + f2hi(a);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    // epilogue: O * delta_v / l -> 16-bit, staged in this block's output tile, TMA store
    bool ep_ok = ok && n_kv > 0;
    if (ep_ok) ep_ok = mbar_wait(&pv_done[t], (gt + n_kv - 1) & 1, abort_flag, kKernFwdFp8, t, 2);
    ep_ok = __all_sync(0xffffffffu, ep_ok);
    // the previous pair's store has read the staging tile (its storing
    // thread waited for that before reaching this barrier)
    if (it > 0) named_barrier_sync(1 + t, 128);
    if (ep_ok) {
      tc_fence_after();
      const float f = p.delta_v / l_sum;
      const uint64_t f2 = f2pack(f, f);
#pragma unroll
      for (int c = 0; c < 128; c += 32) {
        uint32_t o[32];
        tmem_ld32(tm_O + c, o);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint64_t v = mul2(f2pack(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), f2);
          pk[i] = pack2<OUT_BF16>(f2lo(v), f2hi(v));
        }
        // columns c..c+31 = 4 chunks of 16 B in box c/64, logical chunk (c%64)/8 + u
        uint8_t* row_base = sOt + (c / 64) * L::kOutBoxBytes + r * 128;
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
    // every thread of the warpgroup reaches this barrier, whatever happened above
    named_barrier_sync(1 + t, 128);
    if (r == 0 && !*abort_flag) {
      for (int c = 0; c < 2; ++c)
        tma_store_3d(&p.tm_o, sOt + c * L::kOutBoxBytes, c * 64, qtile * 128, bh);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
    ok = ok && ep_ok;
    gt += n_kv;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
