/*
 * fa.h - C ABI of the B200 (sm_100a) exact-attention library libfa_b200.so.
 *
 * The library computes exact softmax attention and its gradient, tiled so
 * that the N x N score matrix never reaches device memory:
 *
 *   forward   O = softmax(scale * Q K^T + causal mask) V, plus one logsumexp
 *             per query row.  The pages define attention as S = QK^T,
 *             P = softmax(S), O = PV ("flash attention io aware", section
 *             "The Memory Bandwidth Bottleneck") and the method as tiles of
 *             Q, K, V streamed through on-chip memory with a running max and
 *             sum, writing only O back ("FlashAttention" glossary, opening
 *             list and online-softmax paragraph; "flash attention io
 *             aware", section "Flash Attention Algorithm").
 *   backward  dQ, dK, dV from Q, K, V, O, dO and the logsumexp alone: the
 *             scores are recomputed on chip instead of being stored
 *             ("FlashAttention" glossary, recomputation paragraph).  dK and
 *             dV are owned by one thread block per key block and written
 *             once, with no atomics ("FlashAttention" glossary,
 *             FlashAttention-2 list, backward-pass item).
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major, in device memory owned by the caller:
 *       q, o, dout, dq : [B][Hq][N][d]
 *       k, v, dk, dv   : [B][Hkv][N][d]
 *       lse            : [B][Hq][N] fp32, natural log:
 *                        lse_i = ln sum_j exp(scale * q_i . k_j) over unmasked j
 *   - Grouped-query attention: Hq % Hkv == 0 and query head h reads key/value
 *     head h / (Hq / Hkv) ("Flash Attention" glossary of inferensys,
 *     grouped-query attention paragraph; Hkv == Hq is plain multi-head,
 *     Hkv == 1 multi-query).  dK and dV sum over each group.
 *   - causal != 0 masks key j for query i when j > i.
 *   - q, k, v, dout share one dtype (bf16 or fp16); o, dq, dk, dv are written
 *     in it.  Arithmetic: tensor-core products of the I/O dtype with fp32
 *     accumulation; softmax statistics in fp32.  (fa_fwd_fp8 alone takes
 *     8-bit E4M3 inputs and a separate output dtype; see there.)
 *   - d must be 64 or 128 (128 for fa_fwd_fp8); N may be any size >= 0 (a ragged last tile is
 *     masked); B == 0 or N == 0 is an empty problem and returns FA_OK at once.
 *   - scale must be finite and > 0 (usually 1/sqrt(d)).
 *   - Every tensor pointer must be 16-byte aligned (TMA requirement).
 *   - stream is a cudaStream_t (NULL: the legacy default stream).  All work is
 *     enqueued asynchronously on it; the call returns without waiting.
 *   - Argument errors are returned before anything is launched.  Errors
 *     inside a kernel (a barrier wait that ran out, see fa_get_device_status)
 *     are recorded on the device; no call aborts the process and there is no
 *     CPU fallback.
 *   - The library never allocates device memory.  Its only state is one
 *     status word per device and a cache of kernel attributes.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, Hq % Hkv != 0, bad scale, small workspace */
    FA_ERR_UNSUPPORTED = 2,  /* d not in {64, 128}, dtype not bf16/fp16, no sm_100 device */
    FA_ERR_MISALIGNED = 3,   /* a tensor pointer is not 16-byte aligned */
    FA_ERR_CUDA = 4,         /* a CUDA runtime or driver call failed */
    FA_ERR_TIMEOUT = 5       /* a kernel's bounded barrier wait ran out (device-side) */
} fa_status_t;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype_t;

/*
 * Forward pass.  Writes o [B][Hq][N][d] and lse [B][Hq][N].
 * Reads q, k, v only; o and lse may not alias the inputs.
 */
fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                   fa_dtype_t dtype, void* stream);

/*
 * Causal sliding-window forward pass: query i attends to keys
 * max(0, i - window + 1) .. i only (window >= 1 keys, itself included; a
 * window of N or more is the plain causal pass).  This banded mask is the
 * simplest block-sparse pattern ("FlashAttention" glossary, block-sparse
 * entry: skip the blocks a sparsity mask hides): key blocks wholly outside
 * the band are not read at all.  Arguments, layouts and errors as fa_fwd;
 * window < 1 returns FA_ERR_INVALID_ARG.
 */
fa_status_t fa_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Hq, int Hkv, int N, int d, float scale, int window,
                          fa_dtype_t dtype, void* stream);

/*
 * Forward pass with dropout on the attention probabilities (the pages list
 * dropout among the operations the attention kernel fuses: "Flash
 * Attention" glossary, kernel-fusion paragraph; they give no rule, this is
 * the library's): inverted dropout with an 8-bit threshold t = round(256 *
 * p_drop): key j of query i is dropped when byte j%4 of word i%4 of
 * Philox4x32-10(counter (j/4, i/4, b*Hq + h, 0), key (seed low 32 bits,
 * seed high 32 bits)) is below t; kept probabilities are scaled by
 * 256 / (256 - t), so the drop rate is exactly t/256.  lse is that of the
 * undropped softmax.  The same (p_drop, seed) must be given to
 * fa_bwd_dropout.  p_drop < 0, not finite, or with t > 255 returns
 * FA_ERR_INVALID_ARG; t = 0 is the plain pass.  Otherwise as fa_fwd.
 */
fa_status_t fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                           float p_drop, uint64_t seed, fa_dtype_t dtype, void* stream);

/*
 * FP8 forward ("FlashAttention" glossary, FlashAttention-3 paragraph: attention
 * on FP8 tensor cores; the pages give no rule, so the plainest one is taken).
 * q [B][Hq][N][128], k and v [B][Hkv][N][128] hold 8-bit E4M3 codes (sign,
 * 4-bit exponent with bias 7, 3-bit fraction; the value of code x times its
 * factor is the input), one factor per tensor: descale_q, descale_k,
 * descale_v.  Computes the forward of fa_fwd on the dequantised inputs:
 *   s_ij = scale * descale_q * descale_k * sum_c q_ic k_jc   (masked as fa_fwd)
 *   O_i  = descale_v * sum_j softmax(s_i.)_j v_j,   lse_i = logsumexp_j s_ij
 * Both products run on E4M3 tensor-core operands with fp32 accumulation; the
 * probabilities are rounded to E4M3 (relative error up to 2^-4 each) for the
 * second product and the row sums are kept in fp32, so lse carries only the
 * fp32 rounding of the 16-bit pass while O carries the E4M3 rounding of P.
 * o [B][Hq][N][128] is written in out_dtype (FA_BF16 or FA_FP16); lse is fp32
 * natural log.  Pointers are caller-owned device memory, 16-byte aligned.
 * Errors: as fa_fwd; a factor that is not finite and > 0 (or whose product
 * with scale overflows fp32) returns FA_ERR_INVALID_ARG; d != 128 returns
 * FA_ERR_UNSUPPORTED.  No backward pass goes with it.
 */
fa_status_t fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int Hq, int Hkv, int N, int d, float scale, float descale_q,
                       float descale_k, float descale_v, int causal, fa_dtype_t out_dtype,
                       void* stream);

/*
 * Bytes of device scratch that fa_bwd needs for these sizes (0 for an empty
 * problem).  Linear in N: two fp32 values per query row (D_i = dO_i . O_i and
 * the logsumexp in base 2) plus an fp32 dQ accumulator [B][Hq][Np][d], with N
 * rounded up to a multiple of 128 (Np), plus 256 bytes (the main pass's
 * work-item counter): 4 * B * Hq * Np * (2 + d) + 256.
 */
size_t fa_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d);

/*
 * Backward pass: given dout = dL/dO, writes dq, dk, dv.  o and lse must be
 * the forward outputs for the same q, k, v, scale and causal flag.  The
 * scores and probabilities are recomputed from q, k and lse.  workspace is
 * caller-owned device memory of at least fa_bwd_workspace_bytes(...) bytes,
 * 16-byte aligned; its contents on entry do not matter and on exit are
 * unspecified.  Three kernels run on `stream` in order: a row pass (D and the
 * zeroed dQ accumulator), the main pass (persistent, one thread block per
 * SM, each taking work items = (key block of 128 rows, key/value head) in
 * turn: dK, dV in tensor memory, dQ added into the accumulator), and a pass
 * that scales and converts dQ.
 */
fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv,
                   int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                   fa_dtype_t dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass of fa_fwd_window (same window); o and lse must come from
 * fa_fwd_window with the same window.  Arguments, workspace, layouts and
 * errors as fa_bwd; window < 1 returns FA_ERR_INVALID_ARG.
 */
fa_status_t fa_bwd_window(const void* q, const void* k, const void* v, const void* o,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv,
                          int B, int Hq, int Hkv, int N, int d, float scale, int window,
                          fa_dtype_t dtype, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * Backward pass of fa_fwd_dropout (same p_drop and seed: the dropout mask is
 * regenerated, not stored).  Otherwise as fa_bwd.
 */
fa_status_t fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv,
                           int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                           float p_drop, uint64_t seed, fa_dtype_t dtype, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * Block-sparse attention ("FlashAttention" glossary, block-sparse entry:
 * blocks that a sparsity mask hides are skipped whole; the page gives no
 * block size or pattern).  block_mask is device memory of bytes over blocks
 * of 128 query rows x 128 keys, nb = ceil(N / 128) blocks a side:
 * [Hq][nb][nb] when mask_per_head = 1, or one [nb][nb] mask for every query
 * head when mask_per_head = 0 (the same mask for every batch entry).  Byte
 * (h, i, j) nonzero: query block i of query head h sees key block j; zero:
 * the whole block is hidden, and nothing of it is computed.  Combined with
 * the causal mask when causal = 1 (a key is seen only if both allow it).  A
 * query row that sees no key at all gets O = 0 and lse = -inf (the log of an
 * empty sum) and adds nothing to the gradients.  The mask is read during
 * the call only.  Limits: Hq / Hkv <= 16 and nb <= 4096, otherwise
 * FA_ERR_UNSUPPORTED; a null mask or mask_per_head outside {0, 1} is
 * FA_ERR_INVALID_ARG.  Otherwise as fa_fwd.
 */
fa_status_t fa_fwd_blockmask(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                             const uint8_t* block_mask, int mask_per_head, fa_dtype_t dtype,
                             void* stream);

/*
 * Workspace of fa_bwd_blockmask: that of fa_bwd plus, per work item (kv head
 * x key block), its step count and the list of (group head, query block)
 * pairs that see it: fa_bwd_workspace_bytes(...) + 4 * B * Hkv * nb
 * + 2 * B * Hkv * nb * (Hq / Hkv) * nb bytes, nb = ceil(N / 128).  0 for an
 * empty problem or Hq % Hkv != 0.
 */
size_t fa_bwd_blockmask_workspace_bytes(int B, int Hq, int Hkv, int N, int d);

/*
 * Backward pass of fa_fwd_blockmask with the same mask: each key block walks
 * only the query blocks that see it (a list made by a planning pass at the
 * start of the call).  o and lse must come from fa_fwd_blockmask; workspace
 * of at least fa_bwd_blockmask_workspace_bytes(...) bytes.  Otherwise as
 * fa_bwd.
 */
fa_status_t fa_bwd_blockmask(const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, void* dq, void* dk, void* dv,
                             int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                             const uint8_t* block_mask, int mask_per_head, fa_dtype_t dtype,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode over a paged key/value cache ("Paper digest: FlashAttention",
 * section "Limits": decode-time attention over a KV cache; "Flash Attention"
 * glossary, PagedAttention entry: the cache lives in fixed-size blocks found
 * through a table).  Sequence b holds L = seq_lens[b] cached tokens, the last
 * Nq of which are the new queries: query t (position L - Nq + t) attends to
 * keys 0 .. L - Nq + t.  Key k of sequence b is slot k % page_size of
 * physical page block_table[b][k / page_size].
 *   q        [B][Hq][Nq][d]                   o   [B][Hq][Nq][d] (same dtype)
 *   k_cache, v_cache [num_pages][Hkv][page_size][d]   lse [B][Hq][Nq] fp32
 *   block_table [B][max_pages] int32 (entries beyond a sequence's pages are
 *   not read), seq_lens [B] int32; all device memory, caller-owned.
 * The work is split along each sequence's pages and merged by logsumexp;
 * workspace (device, 16-byte aligned) holds the partial results:
 * fa_decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_pages) bytes.
 * Supported: d in {64, 128}, page_size in {16, 32, 64, 128},
 * (Hq / Hkv) * Nq <= 32, bf16/fp16.  Host-side errors as fa_fwd; a
 * seq_lens entry outside [Nq, max_pages * page_size] or a block-table
 * entry outside [0, num_pages) is detected on the device (nothing out of
 * range is read) and reported by fa_get_device_status as FA_ERR_INVALID_ARG.
 * Two kernels run on `stream`, launched as programmatic dependents of the
 * work before them: each may be scheduled while the previous kernel on the
 * stream still runs, and waits for it to complete before reading or writing
 * any global memory, so stream order holds as for a plain launch.
 */
size_t fa_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int d, int max_pages);
fa_status_t fa_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                            const int* block_table, const int* seq_lens, void* o, float* lse,
                            int B, int Hq, int Hkv, int Nq, int d, int page_size, int max_pages,
                            int num_pages, float scale, fa_dtype_t dtype, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream`, then returns and clears the first device-side error
 * any kernel of this library recorded on the current device since the last
 * call: FA_OK, or FA_ERR_TIMEOUT when a bounded barrier wait ran out (the
 * kernel then skipped its remaining work and its outputs are undefined), or
 * FA_ERR_INVALID_ARG when fa_decode_paged met a bad table entry or length.
 * Returns FA_ERR_CUDA when the stream itself reports an error.
 */
fa_status_t fa_get_device_status(void* stream);

/*
 * Raw form of the last recorded device status word (0 = none), for
 * diagnostics: bits 0-7 status, 8-15 kernel id, 16-23 warp role, 24-31 wait
 * site.  Does not clear it.  Synchronises `stream`.
 */
uint32_t fa_peek_device_status_word(void* stream);

/*
 * Self-test of the failure path: launches one thread block that waits on a
 * barrier nobody signals, with the wait limit set to limit_ns nanoseconds,
 * then restores the default limit (2 s) and returns what
 * fa_get_device_status reports (FA_ERR_TIMEOUT when the bounded wait works).
 * No fault, trap or hang is involved.
 */
fa_status_t fa_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/*
 * Profiling hook: while set, every launch of kernel `kernel_id` (1: the
 * forward kernel of fa_fwd, 3: the main kernel of fa_bwd) is bracketed by
 * cudaEventRecord(start) / cudaEventRecord(stop) on the stream it is launched
 * on.  start and stop are cudaEvent_t handles created by the caller; pass
 * NULL for both to clear.  Process-wide, not synchronised with concurrent
 * calls: set it only from the thread that launches.
 */
fa_status_t fa_set_profile_events(int kernel_id, void* start, void* stop);

/*
 * Caps the number of thread blocks of fa_bwd's main pass, which otherwise
 * runs one persistent block per SM; each block then takes more work items in
 * turn.  0 restores the default.  Results do not depend on the cap (beyond
 * the order of the fp32 dQ additions); it exists to exercise and measure the
 * hand-over between work items on small problems.  Process-wide; negative
 * values return FA_ERR_INVALID_ARG.
 */
fa_status_t fa_set_bwd_max_blocks(int max_blocks);

/*
 * Backward pass for callers that cannot allocate device memory.
 *
 * fa_bwd needs a caller-provided workspace.  Some callers cannot obtain one:
 * code that runs where cudaMalloc is not allowed or not wanted (a host
 * callback or plugin that only receives raw tensor pointers from a host
 * framework, a real-time loop that forbids allocation after start-up, or a
 * runtime whose memory is owned by another allocator).  This entry point
 * takes the same tensors as fa_bwd but no workspace: it uses a fixed scratch
 * array of FA_BWD_NOALLOC_SCRATCH_BYTES bytes that the library reserves in
 * device memory of every GPU that loads it, kept until the process exits.
 * The pages describe no counterpart; this is an interface convenience.
 *
 * - Size limit: the problem must satisfy
 *     fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) <= FA_BWD_NOALLOC_SCRATCH_BYTES,
 *   otherwise FA_ERR_UNSUPPORTED is returned and nothing is launched.
 * - The first call on a device looks up the array's device address (once
 *   per device, with that device current); make that first call before any
 *   stream capture.  Later calls do no set-up.
 * - No allocation of any kind: no cudaMalloc / cudaFree, no library routine
 *   that allocates.
 * - Every call on a device shares the one array.  Calls whose kernels
 *   overlap on the GPU (different streams, or different host threads without
 *   ordering) race on it and give wrong results: order them on one stream.
 *   The array keeps the last call's contents; each call clears what it needs
 *   zeroed (the dQ accumulator) and overwrites the rest before reading it.
 * - Everything else (arguments, layouts, errors, asynchrony) is as fa_bwd.
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

fa_status_t fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv,
                           int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                           fa_dtype_t dtype, void* stream);

/* Static English description of a status code. */
const char* fa_status_string(fa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
