// Forward pass of exact attention on sm_100a: one thread block per
// (batch, query head, couple of query pairs), a query pair being two
// 128-row query blocks.
//
// Method (pages: "FlashAttention" glossary, opening list and online-softmax
// paragraph; "flash attention io aware", sections "Flash Attention
// Algorithm" and "Online Softmax"): the query blocks stay on chip while the
// key/value blocks of their head stream through a shared-memory ring; each
// score block S_j = Q K_j^T lives only in tensor memory; a running row max m
// and row sum l are kept and the partial output is rescaled when the max
// grows; only O and one logsumexp per row are written back.  Queries are the
// outer loop and key/value blocks the inner one, as in the "Flash Attention"
// glossary of inferensys ("for each query block, iterate over key-value
// blocks"); the other order on the chipfoundry page reaches the same result.
//
// Two query blocks per thread block, each with its own softmax warpgroup, so
// that the tensor cores work on one block while the softmax warps work on the
// other (the B200 form of the "two sets of registers" alternation the
// FlashAttention glossary names for Hopper).  Warp roles (384 threads):
//   warps 0-3 / 4-7  softmax of query block 0 / 1: thread r owns row r of its
//              block and tensor-memory lane r.  Reads S_j, masks, scales,
//              updates (m, l), writes P_j (16-bit) over S_j, rescales O when
//              needed, and at the end of a pair normalises O and writes it
//              and lse (each thread its row).
//   warp 8     MMA issuer (whole warp, one elected lane issues): S_t,j = Q_t K_j^T
//              and O_t += P_t,j V_j
//              for t = 0, 1, staggered as S0_j+1, O1 += P1_j V_j, S1_j+1,
//              O0 += P0_j+1 V_j+1, ... so that one block's softmax overlaps the
//              other block's products.
//   warp 9     TMA producer: Q0, Q1 of a pair, then K_0, V_0, K_1, V_1, ...
//              through a ring of kSlots tiles; then the next pair's.
//   warps 10-11 idle (they complete the third warpgroup, which gives its
//              registers to the softmax warpgroups).
// Tensor memory (512 columns x 128 lanes x 32 bit): S0 [0,128), S1 [128,256),
// O0 [256, 256+d), O1 [384, 384+d); P_t packs into the first 64 columns of S_t.
//
// Running max: the max used for the exponentials (m_ref) moves only when a
// row's max exceeds it by more than kRefSlack = 14 (log2 units), so O and l
// are rescaled rarely, even for wide logits; P = 2^(s - m_ref) <= 2^14 stays
// four times inside the fp16 range (65504), and far inside bf16's.  O and
// l always share one m_ref, so O / l is exact (a softmax's reference point is
// arbitrary).
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace fa {

struct FwdParams {
  CUtensorMap tm_q;  // [B*Hq][N][d], box 64 x 128
  CUtensorMap tm_k;  // [B*Hkv][N][d]
  CUtensorMap tm_v;
  void* o;           // [B*Hq][N][d], written by the softmax threads
  float* lse;        // [B*Hq][N]
  int N, Hq, Hkv, group, BH, n_pairs, n_ktiles;
  int fold;          // 1: a block runs query pairs n-1-c and c; 0: one pair
  int window;        // causal sliding window of this many keys (query i sees i-W+1..i); 0: none
  // dropout (kernels instantiated with DROP): key j of query i is dropped
  // when byte j%4 of word i%4 of Philox4x32-10((j/4, i/4, bh, 0), seed) is
  // below drop_t; kept probabilities are scaled by drop_scale = 256/(256-t)
  uint32_t seed_lo, seed_hi, drop_t;
  float drop_scale;
  float scale_log2;  // scale * log2(e)
  // block mask (kernels instantiated with BMASK): key block j (128 keys) is
  // hidden from query block i (128 rows) of query head h when
  // bmask[h * bm_hstride + i * n_ktiles + j] == 0 (bm_hstride 0: one mask
  // for every head)
  const uint8_t* bmask;
  long long bm_hstride;
};

// The key blocks a pair of query blocks streams under a block mask: those
// visible to either block (union), in order.  Block t of the pair sees key
// block j when j <= jmax[t] (causal) and its mask byte is set.
struct FwdMaskRows {
  // mask rows of the pair's query blocks (nullptr: no such block); the
  // fields are named, not an array, so that a runtime t selects by value
  const uint8_t* row0;
  const uint8_t* row1;
  int jmax0, jmax1;

  __device__ __forceinline__ bool vis(int t, int j) const {
    const uint8_t* r = t ? row1 : row0;
    return r != nullptr && j <= (t ? jmax1 : jmax0) && __ldg(r + j) != 0;
  }
  __device__ __forceinline__ int jend() const { return max(jmax0, jmax1) + 1; }
  // first key block >= j that either block sees; jend() if none
  __device__ __forceinline__ int next(int j) const {
    const int e = jend();
    while (j < e && !vis(0, j) && !vis(1, j)) ++j;
    return j;
  }
  // number of key blocks in the union, counted by the whole warp
  __device__ __forceinline__ int count_warp(int lane) const {
    int n = 0;
    for (int j0 = 0; j0 < jend(); j0 += 32) {
      const int j = j0 + lane;
      n += __popc(__ballot_sync(0xffffffffu, j < jend() && (vis(0, j) || vis(1, j))));
    }
    return n;
  }
};

template <int HD>
struct FwdLayout {
  static constexpr int kBoxBytes = 128 * 128;        // 128 rows x 64 columns x 2 B
  static constexpr int kChunks = HD / 64;            // 64-column boxes per tile
  static constexpr int kTileBytes = 128 * HD * 2;    // one 128-row tile
  static constexpr int kSlots = HD == 128 ? 5 : 8;   // K/V ring depth
  static constexpr int kOffQ = 0;                    // two query tiles
  static constexpr int kOffRing = 2 * kTileBytes;
  static constexpr int kOffBar = kOffRing + kSlots * kTileBytes;
  // barriers: q_full, slot_full[kSlots], slot_empty[kSlots], s_full[2],
  // p_half[2][2] (keys 0-63 / 64-127 of P_t ready), pv_done[2], done, q_free
  static constexpr int kNumBars = 1 + 2 * kSlots + 8 + 1 + 1;
  static constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemPtr + 4;
  static constexpr int kSmemBytes = kOffAbort + 4;
  static constexpr int kDynSmem = kSmemBytes + 1024;  // slack for 1024-byte alignment
  static_assert(kDynSmem <= 232448, "shared memory budget");
};

// Three warpgroups: two softmax warpgroups and one holding the MMA issuer,
// the TMA producer and two idle warps.  Launched at 168 registers a thread
// (384 x 168 of the SM's 65 536), the registers are then moved to the
// softmax warpgroups: 2 x 128 x 208 + 128 x 88 = 384 x 168.  Per SM
// sub-partition (16 384 registers, one warp of each warpgroup) that is
// 32 x (208 + 208 + 88) = 16 128.  (216 / 72 left the MMA and TMA warps
// spilling; 208 suffices for the softmax warps.)
constexpr int kFwdThreads = 384;
constexpr uint32_t kFwdSoftmaxRegs = 208;
constexpr uint32_t kFwdOtherRegs = 88;
static_assert(2 * 128 * kFwdSoftmaxRegs + 128 * kFwdOtherRegs <= kFwdThreads * 168, "register split");
constexpr uint32_t kKernFwd = 1;
// How far a row's max may run above the reference max of its exponentials
// (log2 units) before the reference moves (O and l rescaled, the tile
// redone): 12 rather than 8 measured 3 % faster, 14 another 1.4 %, on
// 64K-token rows with wide logits, which move the reference less often.
constexpr float kRefSlack = 14.0f;
// One query pair of a head: its two 128-row query blocks and the key blocks
// they stream.
struct FwdItem {
  int bh, pair, kvh, j_start, n_kv0, n_kv1;
  FwdMaskRows mrows;
};

template <bool CAUSAL, bool BMASK>
__device__ __forceinline__ FwdItem fwd_item(const FwdParams& p, int bh, int pair) {
  FwdItem it;
  it.bh = bh;
  it.pair = pair;
  const int h = bh % p.Hq;
  const int b = bh / p.Hq;
  it.kvh = b * p.Hkv + h / p.group;
  // key blocks seen by query block t (t = 0, 1) of the pair.  With a sliding
  // window the key/value stream starts at the first block the pair's first
  // row can see; counts are of blocks from that one on.
  it.j_start = (CAUSAL && p.window > 0) ? max(0, 2 * pair * 128 - p.window + 1) / 128 : 0;
  it.n_kv0 = (CAUSAL ? min(2 * pair + 1, p.n_ktiles) : p.n_ktiles) - it.j_start;
  it.n_kv1 = (CAUSAL ? min(2 * pair + 2, p.n_ktiles) : p.n_ktiles) - it.j_start;
  // Under a block mask both blocks walk the union of their visible key
  // blocks (n_kv0 = n_kv1 = its size, counted by each role's warp); a key
  // block hidden from one of them is a fully masked tile for it.
  it.mrows = FwdMaskRows{};
  if constexpr (BMASK) {
    const uint8_t* mh = p.bmask + static_cast<long long>(h) * p.bm_hstride;
    const int qb0 = 2 * pair, qb1 = 2 * pair + 1;
    it.mrows.row0 = mh + static_cast<long long>(qb0) * p.n_ktiles;
    it.mrows.row1 = qb1 < p.n_ktiles ? mh + static_cast<long long>(qb1) * p.n_ktiles : nullptr;
    it.mrows.jmax0 = CAUSAL ? min(qb0, p.n_ktiles - 1) : p.n_ktiles - 1;
    it.mrows.jmax1 = CAUSAL ? min(qb1, p.n_ktiles - 1) : p.n_ktiles - 1;
  }
  return it;
}

template <int HD, bool BF16, bool CAUSAL, bool DROP, bool BMASK>
__global__ void __launch_bounds__(kFwdThreads, 1) fa_fwd_kernel(const __grid_constant__ FwdParams p) {
  static_assert(!(DROP && BMASK), "dropout and block masks are not combined");
  using L = FwdLayout<HD>;
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
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
  uint64_t* p_half = s_full + 2;  // [t][half]
  uint64_t* pv_done = p_half + 4;
  uint64_t* done_bar = pv_done + 2;
  uint64_t* q_free = done_bar + 1;  // every S product of a pair (the readers of sQ) has completed
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sm + L::kOffTmemPtr);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kOffAbort);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // The block's work: query pairs n-1-c and c of head bh, back to back (one
  // pair when they coincide).  Under a causal mask pair i streams 2i + 2 key
  // blocks, so every couple has the same length and the blocks of a launch
  // take equal time; the second pair's Q load and first S product overlap
  // the first pair's last tiles and epilogue.  Head-major order: the blocks
  // running at the same time mostly share a head, so its K and V stay in L2.
  // Without folding (long sequences, where a pair's fixed costs are small
  // next to its key blocks) a block runs one pair, the longest first.
  const int n_couples = p.fold ? (p.n_pairs + 1) / 2 : p.n_pairs;
  const int bh = blockIdx.x / n_couples;
  const int cpl = blockIdx.x % n_couples;
  const int n_items = (!p.fold || p.n_pairs - 1 - cpl == cpl) ? 1 : 2;
  auto item_pair = [&](int it) { return it == 0 ? p.n_pairs - 1 - cpl : cpl; };

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    for (int s = 0; s < L::kSlots; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_half[2 * i], 128);
      mbar_init(&p_half[2 * i + 1], 128);
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
  // Each warpgroup changes its register count at one site, all four of its
  // warps together (the PTX rule for setmaxnreg); the roles branch below it.
  if (warp >= 8) setmaxnreg_dec<kFwdOtherRegs>();
  if (warp >= 10) {
    // idle warps of the third warpgroup
  } else if (warp == 9) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&p.tm_q);
      prefetch_tensormap(&p.tm_k);
      prefetch_tensormap(&p.tm_v);
    }
    int n = 0;  // K/V tiles loaded (ring position), over both pairs
    bool ok = true;
    for (int it = 0; ok && it < n_items; ++it) {
      const FwdItem I = fwd_item<CAUSAL, BMASK>(p, bh, item_pair(it));
      int n_kv1 = I.n_kv1;
      if constexpr (BMASK) n_kv1 = I.mrows.count_warp(lane);
      if (lane == 0) {
        // Q0, Q1 of the pair; the previous pair's S products, the last
        // readers of sQ, must have completed
        if (it > 0) ok = mbar_wait(q_free, (it - 1) & 1, abort_flag, kKernFwd, 9, 1);
        if (ok) {
          mbar_expect_tx(q_full, 2 * L::kTileBytes);
          for (int t = 0; t < 2; ++t)
            for (int c = 0; c < L::kChunks; ++c)
              tma_load_3d(sQ + t * L::kTileBytes + c * L::kBoxBytes, &p.tm_q, q_full, c * 64,
                          (2 * I.pair + t) * 128, I.bh);
          // the next pair's Q into L2 now, so that its load (which must wait
          // for this pair's last S product) finds it there
          if (it + 1 < n_items)
            for (int t = 0; t < 2; ++t)
              if ((2 * item_pair(it + 1) + t) * 128 < p.N)
                for (int c = 0; c < L::kChunks; ++c)
                  tma_prefetch_3d(&p.tm_q, c * 64, (2 * item_pair(it + 1) + t) * 128, I.bh);
        }
        auto load = [&](const CUtensorMap* map, int kblock) -> bool {
          const int s = n % L::kSlots;
          if (n >= L::kSlots &&
              !mbar_wait(&slot_empty[s], ((n / L::kSlots) - 1) & 1, abort_flag, kKernFwd, 9, 0))
            return false;
          mbar_expect_tx(&slot_full[s], L::kTileBytes);
          uint8_t* dst = sRing + s * L::kTileBytes;
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_3d(dst + c * L::kBoxBytes, map, &slot_full[s], c * 64, kblock * 128, I.kvh);
          ++n;
          return true;
        };
        int kb = BMASK ? I.mrows.next(0) : I.j_start;  // key block of stream position j
        for (int j = 0; ok && j < n_kv1; ++j) {
          ok = load(&p.tm_k, kb);
          if (ok) ok = load(&p.tm_v, kb);
          kb = BMASK ? I.mrows.next(kb + 1) : kb + 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop with warp-uniform values; one elected
    // lane issues each MMA and commit.  Descriptors are formed once and
    // moved by constant offsets.
    constexpr uint32_t kIdS = idesc_f16(BF16, 128, 128, false, false);
    constexpr uint32_t kIdPV = idesc_f16(BF16, 128, HD, false, true);
    const uint64_t dQ_k = sdesc_sw128(smem_u32(sQ), 16, 1024);           // Q tile 0, K-major
    const uint64_t dR_k = sdesc_sw128(smem_u32(sRing), 16, 1024);        // ring slot 0, K-major
    const uint64_t dR_mn = sdesc_sw128(smem_u32(sRing), L::kBoxBytes, 1024);  // ring slot 0, MN-major
    auto wait_all = [&](uint64_t* bar, uint32_t parity, uint32_t site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, kKernFwd, 8, site));
    };
    int n = 0;  // K/V tiles taken from the ring, over both pairs
    auto take = [&](int& slot) -> bool {
      slot = n % L::kSlots;
      if (!wait_all(&slot_full[slot], (n / L::kSlots) & 1, 1)) return false;
      tc_fence_after();
      ++n;
      return true;
    };
    // Staggered order: S0_0 S1_0 PV0_0 | S0_1 PV1_0 S1_1 PV0_1 | S0_2 PV1_1 ...
    // so that one block's softmax runs while the tensor cores work on the
    // other block.  K_j and V_j are taken in load order (K0 V0 K1 V1 ...).
    // S_t,j+1 is written over the tensor memory that O_t += P_t,j V_j reads
    // P_t,j from, and is issued right after it by this same warp: the tensor
    // core runs the MMAs of one thread in issue order, reading an MMA's
    // operands before a later MMA writes its result, so no wait is put
    // between them (waiting for an MMA's completion before issuing the next
    // costs several hundred cycles of idle tensor core on B200).  The same
    // holds across the two pairs: the next pair's S_t,0 follows the last
    // O_t += P_t V.
    auto issue_s = [&](int t, int kslot) {
      const uint32_t qo = t * L::kTileBytes, ko = kslot * L::kTileBytes;
#pragma unroll
      for (int k = 0; k < HD / 16; ++k) {
        const uint32_t off = (k >> 2) * L::kBoxBytes + (k & 3) * 32;
        umma_ss_w(tmem + t * 128, sdesc_add(dQ_k, qo + off), sdesc_add(dR_k, ko + off), kIdS, k > 0);
      }
      umma_commit_w(&s_full[t]);
    };
    // O_t += P_t,j V_j in two halves of 64 keys: the softmax warps hand over
    // P of keys 0-63 before they compute keys 64-127.  g: the tile's index
    // over both pairs (barrier phase), j: its index in the pair.
    auto issue_pv = [&](int t, int g, int j, int vslot) -> bool {
      const uint32_t vo = vslot * L::kTileBytes;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        if (!wait_all(&p_half[2 * t + half], g & 1, 3)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 4 * half; k < 4 * half + 4; ++k)
          umma_ts_w(tmem + 256 + t * 128, tmem + t * 128 + k * 8, sdesc_add(dR_mn, vo + k * 2048),
                    kIdPV, (j > 0 || k > 0) ? 1u : 0u);
      }
      umma_commit_w(&pv_done[t]);
      return true;
    };
    int g0 = 0, g1 = 0;  // tiles of query block 0 / 1 in the pairs before this one
    bool ok = true;
    for (int it = 0; ok && it < n_items; ++it) {
      const FwdItem I = fwd_item<CAUSAL, BMASK>(p, bh, item_pair(it));
      int n_kv0 = I.n_kv0, n_kv1 = I.n_kv1;
      if constexpr (BMASK) n_kv0 = n_kv1 = I.mrows.count_warp(lane);
      if (!(ok = wait_all(q_full, it & 1, 0))) break;
      tc_fence_after();
      if (n_kv1 == 0) {
        // nothing to compute (only under a block mask): sQ is free at once
        umma_commit_w(q_free);
        continue;
      }
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
    mbar_wait_drain(done_bar, 0, kKernFwd, 8, 4);
  } else {
    setmaxnreg_inc<kFwdSoftmaxRegs>();
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;                 // query block of this warpgroup
    const int r = tid & 127;                 // row within the block == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tm_S = tmem + t * 128 + lane_off;
    const uint32_t tm_O = tmem + 256 + t * 128 + lane_off;
    const float c_log2 = p.scale_log2;
    const uint64_t c2 = f2pack(c_log2, c_log2);
    int gt = 0;  // tiles of this query block in the pairs before this one
    bool ok = true;
    for (int it = 0; ok && it < n_items; ++it) {
    const FwdItem I = fwd_item<CAUSAL, BMASK>(p, bh, item_pair(it));
    const FwdMaskRows& mrows = I.mrows;
    int n_kv0 = I.n_kv0, n_kv1 = I.n_kv1;
    const int qtile = 2 * I.pair + t;
    const int q_row = qtile * 128 + r;
    if constexpr (BMASK) n_kv0 = n_kv1 = mrows.count_warp(lane);
    const int n_kv = t ? n_kv1 : n_kv0;
    int kb_cur = BMASK ? mrows.next(0) : I.j_start;  // key block of the current stream position
    float m_ref = -INFINITY;  // in log2 units of the scaled scores
    float l_sum = 0.f;
    // Waits are made warp-uniform: tcgen05.ld/st are warp-collective, so a
    // warp either goes on together or leaves together (on abort).
    //
    // Per key tile: S is read from tensor memory, masked where a block edge
    // needs it, and the row max taken (three-input max, eight chains).  From
    // the second tile on, the exponentials of keys 0-63 are computed against
    // the current reference max while the row max is still being taken (the
    // two are independent), so that the max costs no time of its own; the
    // warp then checks whether any of its rows grew by more than kRefSlack (log2).
    // If none did (the common case) those exponentials stand: P of keys 0-63
    // goes to tensor memory and is handed to the MMA warp, then keys 64-127.
    // Otherwise the tile is redone from tensor memory against the moved
    // reference, after O and l are rescaled.
      auto load_s = [&](int kblock, uint32_t* s) {
        tmem_ld32(tm_S + 0, s);
        tmem_ld32(tm_S + 32, s + 32);
        tmem_ld32(tm_S + 64, s + 64);
        tmem_ld32(tm_S + 96, s + 96);
        tmem_ld_wait();
        // mask: keys past the end of the sequence, and keys after the query
        // inside the diagonal block of a causal problem
        const int kv0 = kblock * 128;
        const bool diag = CAUSAL && (kblock == qtile);
        // sliding window: keys below q_row - W + 1 are hidden; some row of the
        // block meets that edge in this key block
        const bool low = CAUSAL && p.window > 0 && kv0 + p.window <= qtile * 128 + 127;
        // block mask: a key block of the pair's stream that this query block
        // does not see is hidden whole
        const bool hid = BMASK && !mrows.vis(t, kblock);
        if (diag || low || hid || kv0 + 128 > p.N) {
          const int lim = hid ? -1 : min(diag ? r : 127, p.N - 1 - kv0);  // last visible column
          const int first = low ? q_row - p.window + 1 - kv0 : 0;  // first visible column
  #pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > lim || c < first) s[c] = __float_as_uint(-INFINITY);
          return true;   // masked tile
        }
        return false;
      };
      // P of the 32 keys 32*q4 .. +31 against the reference -m (nm2), packed to
      // 16 bits in pk[16]; the unrounded values are summed into acc.
      auto p_chunk = [&](const uint32_t* s, int q4, uint64_t nm2, int kv0, uint32_t* pk, uint64_t* acc) {
        [[maybe_unused]] uint32_t kw[4] = {0, 0, 0, 0};  // dropout bytes: keys 4g..4g+3 of 16 in kw[g]
  #pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = q4 * 32 + 2 * i;
          const uint64_t x = fma2(f2pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), c2, nm2);
          const uint64_t pp = f2pack(ex2_approx(f2lo(x)), ex2_approx(f2hi(x)));
          acc[i & 3] = add2(acc[i & 3], pp);  // l sums the undropped P
          if constexpr (DROP) {
            if ((i & 7) == 0) {
              // The 4 lanes of a quad hold 4 consecutive rows (one Philox
              // counter row).  Lane g of the quad draws the 4x4 block of keys
              // 4g..4g+3 of the next 16; four rotations of a shuffle give
              // each lane its own row's word of all four blocks.
              const int ql = lane & 3;
              const uint4 rnd = philox4x32_10(
                  make_uint4(static_cast<uint32_t>((kv0 + c + 4 * ql) >> 2), static_cast<uint32_t>(q_row >> 2),
                             static_cast<uint32_t>(bh), 0u),
                  p.seed_lo, p.seed_hi);
  #pragma unroll
              for (int rr = 0; rr < 4; ++rr) {
                const uint32_t got = __shfl_sync(0xffffffffu, uint4_word(rnd, (ql - rr) & 3),
                                                 (lane & ~3) | ((ql + rr) & 3));
                const int g = (ql + rr) & 3;
                kw[0] = g == 0 ? got : kw[0];
                kw[1] = g == 1 ? got : kw[1];
                kw[2] = g == 2 ? got : kw[2];
                kw[3] = g == 3 ? got : kw[3];
              }
            }
            const uint32_t keep_word = kw[(i >> 1) & 3];
            const uint32_t b0 = (keep_word >> (16 * (i & 1))) & 0xFFu;
            const uint32_t b1 = (keep_word >> (16 * (i & 1) + 8)) & 0xFFu;
            pk[i] = pack2<BF16>(b0 >= p.drop_t ? f2lo(pp) : 0.f, b1 >= p.drop_t ? f2hi(pp) : 0.f);
          } else {
            pk[i] = pack2<BF16>(f2lo(pp), f2hi(pp));
          }
        }
      };
      auto hand_over = [&](int half) {
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_half[2 * t + half]);
      };
      auto sum_acc = [&](const uint64_t* acc) {
        const uint64_t a = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
        return f2lo(a) + f2hi(a);
      };
      for (int j = 0; j < n_kv; ++j) {
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[t], (gt + j) & 1, abort_flag, kKernFwd, t, 0))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kb = kb_cur;
        if constexpr (BMASK) kb_cur = mrows.next(kb + 1);
        else kb_cur = kb + 1;
        const int kv0 = kb * 128;
        bool done = false;
        float m_new;
        {
          uint32_t s[128];
          load_s(kb, s);
          // row max, eight independent chains of three-input maxima: chain i
          // takes columns i, i + 8, ..., i + 120
          float mx[8];
  #pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = fmaxf(__uint_as_float(s[i]), __uint_as_float(s[8 + i]));
  #pragma unroll
          for (int c = 16; c < 128; c += 16)
  #pragma unroll
            for (int i = 0; i < 8; ++i)
              mx[i] = max3f(mx[i], __uint_as_float(s[c + i]), __uint_as_float(s[c + 8 + i]));
          m_new = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * c_log2;
          if (j > 0) {
            // speculative: keys 0-63 against the current reference
            const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
            const uint64_t nm2 = f2pack(-m_use, -m_use);
            uint32_t pk0[16], pk1[16];
            uint64_t acc[4] = {0, 0, 0, 0};
            p_chunk(s, 0, nm2, kv0, pk0, acc);
            p_chunk(s, 1, nm2, kv0, pk1, acc);
            if (!__any_sync(0xffffffffu, m_new > m_ref + kRefSlack)) {
              tmem_st16(tm_S + 0, pk0);
              tmem_st16(tm_S + 16, pk1);
              hand_over(0);
              p_chunk(s, 2, nm2, kv0, pk0, acc);
              tmem_st16(tm_S + 32, pk0);
              p_chunk(s, 3, nm2, kv0, pk1, acc);
              tmem_st16(tm_S + 48, pk1);
              l_sum += sum_acc(acc);
              hand_over(1);
              done = true;
            }
          } else {
            // first tile of the rows: the reference is this tile's max, and
            // the scores are still in registers
            m_ref = m_new;
            const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
            const uint64_t nm2 = f2pack(-m_use, -m_use);
            uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint32_t pk[16];
              p_chunk(s, q4, nm2, kv0, pk, acc);
              tmem_st16(tm_S + q4 * 16, pk);
              if (q4 == 1) hand_over(0);
            }
            l_sum += sum_acc(acc);
            hand_over(1);
            done = true;
          }
        }
        if (done) continue;
        // first tile of the rows, or a reference max that must move
        if (j > 0) {
          // Move the reference max of every row of this warp (tcgen05.ld/st are
          // warp-wide), rescaling O and l, once O_t += P_t,j-1 V_j-1 is done.
          if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[t], (gt + j - 1) & 1, abort_flag, kKernFwd, t, 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float m_upd = fmaxf(m_ref, m_new);
          // rows still without a visible key (m_upd = -inf) keep their zeros
          const float corr = m_upd == -INFINITY ? 1.f : ex2_approx(m_ref - m_upd);
          const uint64_t corr2 = f2pack(corr, corr);
          m_ref = m_upd;
          l_sum *= corr;
  #pragma unroll 1
          for (int c = 0; c < HD; c += 16) {
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
        } else {
          m_ref = m_new;
        }
        {
          // P = 2^(s c - m_ref), packed to 16 bits over the first 64 columns of
          // S.  A row that has seen no visible key yet (only under a sliding
          // window) keeps m_ref = -inf; its scores are all -inf and give P = 0
          // against 0.
          uint32_t s[128];
          load_s(kb, s);
          const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
          const uint64_t nm2 = f2pack(-m_use, -m_use);
          uint64_t acc[4] = {0, 0, 0, 0};
  #pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t pk[16];
            p_chunk(s, q4, nm2, kv0, pk, acc);
            tmem_st16(tm_S + q4 * 16, pk);
            if (q4 == 1) hand_over(0);
          }
          l_sum += sum_acc(acc);
          hand_over(1);
        }
      }
    // epilogue: O / l -> 16-bit, written from registers (each thread its row)
    // no key block at all to stream (only under a block mask): O = 0
    const bool empty_stream = ok && n_kv == 0;
    bool ep_ok = ok && n_kv > 0;
    if (ep_ok) ep_ok = mbar_wait(&pv_done[t], (gt + n_kv - 1) & 1, abort_flag, kKernFwd, t, 2);
    ep_ok = __all_sync(0xffffffffu, ep_ok);
    if (ep_ok || empty_stream) {
      if (ep_ok) tc_fence_after();
      // with dropout, the kept probabilities' factor 1/(1-p) is applied here,
      // once, rather than before P is rounded to 16 bits.  A row that saw
      // no key (possible only under a block mask) has l = 0: O = 0 and
      // lse = -inf, the log of an empty sum.
      const bool seen = l_sum > 0.f;
      const float inv_l = seen ? (DROP ? p.drop_scale : 1.0f) / l_sum : 0.f;
      const uint64_t inv2 = f2pack(inv_l, inv_l);
      T* orow = reinterpret_cast<T*>(p.o) + (static_cast<size_t>(bh) * p.N + q_row) * HD;
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        uint32_t o[32];
        if (ep_ok) {
          tmem_ld32(tm_O + c, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint64_t v = mul2(f2pack(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), inv2);
          pk[i] = pack2<BF16>(f2lo(v), f2hi(v));
        }
        if (q_row < p.N) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(orow + c + 8 * u) =
                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
      if (q_row < p.N)
        p.lse[static_cast<size_t>(bh) * p.N + q_row] =
            seen ? (m_ref + __log2f(l_sum)) * 0.69314718055994531f : -INFINITY;
      // this pair's O has been read: the next pair's first P V may overwrite it
      tc_fence_before();
    }
    ok = ok && (ep_ok || empty_stream);
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
