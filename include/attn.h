/*
 * attn.h - C ABI of the B200 (sm_100a) fused-attention library.
 *
 * The library computes softmax attention,  O = softmax(scale * Q K^T + mask) V,
 * block by block with an online softmax, so that the T x S score matrix never
 * reaches device memory.  That is the FlashAttention scheme of the page
 * "Snelle attention-kernels en operatorfusie versnellen AI-modellen"
 * (the-ai.news), section "FlashAttention-type aandacht en gepagineerde
 * aandacht": queries, keys and values are processed per block; for each block
 * a part of the scores is formed, the softmax statistics (running row maximum
 * and running sum) are updated and the matching output is accumulated in
 * on-chip memory.  The same section defines the paged KV cache served by
 * paged_attn_decode: fixed-size blocks (16 tokens in its example) and a block
 * table that maps every logical position to a physical block.
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 *  - All tensor pointers are DEVICE pointers on the current CUDA device,
 *    allocated, owned and freed by the caller.  The library never frees or
 *    retains them beyond the call's completion on `stream`.
 *  - bf16 tensors are passed as `void*` (IEEE bfloat16, row-major,
 *    contiguous, 16-byte aligned base).  Float outputs are fp32.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; 0 = legacy
 *    default stream) and performs no host<->device synchronisation.
 *  - Kernels are launched as programmatic dependents of the work before them
 *    on `stream`: their set-up (barriers, tensor memory, L2 prefetches of
 *    inputs whose addresses need no memory read) may overlap the previous
 *    kernel's tail, but every read or write of caller memory happens after
 *    that kernel has completed, so stream order is unchanged for the caller.
 *  - Calls on different streams may run at the same time (for example a
 *    prefill on one stream and a decode on another): each call's temporary
 *    memory is allocated and freed in the order of its own stream.  The one
 *    exception is paged_attn_decode_noalloc, whose calls share one scratch
 *    buffer (see there).  The per-device host state is set up once under a
 *    lock, so calls may also come from several host threads.
 *  - Return value: ATTN_OK (0) or a negative attn_status_t.  Argument errors
 *    are detected on the host before anything is launched; nothing is written
 *    to the outputs in that case.  There is no fallback path: an unsupported
 *    shape returns ATTN_ERR_UNSUPPORTED.
 *  - Device-side bounded waits: every wait inside a kernel gives up after a
 *    time limit, records ATTN_DEVSTATUS_TIMEOUT in a device status word and
 *    lets the kernel exit (the outputs of that call are then undefined).
 *    attn_read_device_status() reads (and optionally clears) that word.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (struct CUstream_st*), declared here so that the
 * header does not require the CUDA headers. */
typedef struct CUstream_st* attn_stream_t;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = -1, /* null pointer, negative size, Hq % Hkv != 0, bad scale ... */
  ATTN_ERR_UNSUPPORTED = -2, /* valid but not implemented (head dim, block size, device) */
  ATTN_ERR_CUDA = -3,        /* a CUDA runtime/driver call or a launch failed */
  ATTN_ERR_TIMEOUT = -4      /* reported by attn_read_device_status() only */
} attn_status_t;

/* Bits of the device status word (see attn_read_device_status). */
#define ATTN_DEVSTATUS_TIMEOUT 0x1
/* A paged call met a block-table entry outside the pool: the entry was not
 * read through and its block_size positions were left out of the softmax
 * (their keys masked).  Without a pool size (the unchecked entry points)
 * only negative ids and ids of 2^27 - 1 or more are caught this way. */
#define ATTN_DEVSTATUS_BAD_BLOCK 0x2
/* A paged call met a seq_lens entry below 0 or above max_blocks * block_size
 * (more positions than its table row names): it was clamped into that range. */
#define ATTN_DEVSTATUS_BAD_SEQLEN 0x4

/*
 * attn_fwd - dense prefill attention with grouped-query heads.
 *
 *   q    [B, T, Hq,  d] bf16   queries
 *   k    [B, S, Hkv, d] bf16   keys
 *   v    [B, S, Hkv, d] bf16   values
 *   o    [B, T, Hq,  d] bf16   output (written)
 *   lse  [B, Hq, T]     fp32   per-row log-sum-exp of the scaled scores,
 *                              natural log (written; may be NULL to skip)
 *
 *   Query head h reads key/value head h / (Hq / Hkv) (contiguous groups).
 *   causal != 0: row i sees key j iff j <= i + (S - T) (bottom-right aligned;
 *   the usual j <= i when T == S).  A row that sees no key gets O = 0 and
 *   LSE = -inf.  scale multiplies Q K^T (1/sqrt(d) for standard attention).
 *
 *   Supported: d in {64, 128}; Hq % Hkv == 0; B, T, S >= 0 (T == 0 or
 *   B == 0 is a no-op); sm_100 device.  Pointers 16-byte aligned.
 *   Errors: ATTN_ERR_INVALID_ARG for null pointers, negative sizes,
 *   Hq/Hkv <= 0, Hq % Hkv != 0, non-finite or non-positive scale;
 *   ATTN_ERR_UNSUPPORTED for other head dims, unaligned pointers or a
 *   non-sm_100 device; ATTN_ERR_CUDA if a launch fails.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int Hq, int Hkv, int T, int S, int d, int causal, float scale,
             attn_stream_t stream);

/*
 * attn_fwd_varlen - attn_fwd over packed sequences of different lengths,
 * with no padding (the "dynamic sequence lengths without padding" of the
 * FlashAttention-2 item on the page "内核更新内容一览", section 关键技术点).
 *
 *   q    [total_q, Hq,  d] bf16   the B sequences' queries, back to back
 *   k    [total_k, Hkv, d] bf16   their keys, back to back
 *   v    [total_k, Hkv, d] bf16
 *   o    [total_q, Hq,  d] bf16   (written)
 *   lse  [Hq, total_q]     fp32   (written; may be NULL)
 *   cu_seqlens_q, cu_seqlens_k: device int32 [B + 1] prefix sums: sequence b
 *   owns query rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key rows
 *   [cu_seqlens_k[b], cu_seqlens_k[b+1]); cu_seqlens_*[0] = 0 and
 *   cu_seqlens_*[B] = total_*.  Lengths may differ between q and k and may
 *   be 0.  max_seqlen_q must be >= every query length (rows beyond it are
 *   not computed).
 *
 *   Each sequence is attended on its own with the rules of attn_fwd
 *   (bottom-right causal alignment per sequence with its own T and S, GQA
 *   map, O = 0 / LSE = -inf for rows that see no key).  Keys of other
 *   sequences are never given weight; inputs are assumed finite.
 *   Supported and errors: as attn_fwd; B == 0 or total_q == 0 is a no-op.
 */
int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                    int B, int max_seqlen_q, int total_q, int total_k,
                    int Hq, int Hkv, int d, int causal, float scale, attn_stream_t stream);

/*
 * paged_attn_decode - one query token per sequence against a paged KV cache.
 *
 *   q            [B, Hq, d]                         bf16
 *   k_cache      [num_blocks, block_size, Hkv, d]   bf16  (pool of physical blocks)
 *   v_cache      [num_blocks, block_size, Hkv, d]   bf16
 *   block_table  [B, max_blocks] int32: physical block of logical block j of
 *                sequence b.  Only entries j < ceil(seq_lens[b]/block_size)
 *                are read; they must be valid block ids of the pool (the
 *                pool's size is not an argument here: paged_attn_decode_checked
 *                takes it and masks ids outside it; this entry point catches
 *                only negative ids and ids >= 2^27 - 1, see
 *                ATTN_DEVSTATUS_BAD_BLOCK).
 *   seq_lens     [B] int32: cached tokens of each sequence (0 allowed, which
 *                gives O = 0).  A value below 0 or above
 *                max_blocks * block_size is clamped into that range and sets
 *                ATTN_DEVSTATUS_BAD_SEQLEN; no table entry past the row is
 *                ever read.
 *   o            [B, Hq, d] bf16 (written)
 *
 *   The query of sequence b sits at position seq_lens[b]-1 and sees every
 *   cached token, scale = 1/sqrt(d).  Query head h reads kv head
 *   h / (Hq / Hkv).
 *
 *   num_splits: the logical blocks of each sequence are cut into ranges of
 *   ceil(max_blocks / num_splits) blocks, each handled by its own CTA, and
 *   the partial results are merged with a log-sum-exp combine.  num_splits
 *   <= 0 picks a value that fills the GPU.  The result does not depend on
 *   the physical placement of the blocks (bit-identical for any permutation
 *   of block ids with the same num_splits).
 *
 *   Workspace: partial outputs (num_splits * B * Hq * (d + 1) fp32) come from
 *   a library-owned, stream-ordered memory pool (cudaMallocFromPoolAsync /
 *   cudaFreeAsync on `stream`).
 *
 *   Supported: d in {64, 128}; block_size == 16; 1 <= Hq/Hkv <= 8;
 *   max_blocks < 2^27; sm_100 device; 16-byte aligned q, caches and o.
 *   Errors: as attn_fwd; ATTN_ERR_INVALID_ARG also for max_blocks <= 0 when
 *   B > 0.
 */
int paged_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_table, const int32_t* seq_lens,
                      int B, int Hq, int Hkv, int d, int block_size, int max_blocks,
                      int num_splits, void* o, attn_stream_t stream);

/*
 * paged_attn_decode_checked - paged_attn_decode for a pool of known size.
 *
 * The same translation through the block table ("De aandachtskernel moet
 * dan elke positie via deze tabel vertalen", page "Snelle attention-kernels
 * en operatorfusie versnellen AI-modellen", section "FlashAttention-type
 * aandacht en gepagineerde aandacht"), with every id checked against the
 * pool before it is used.
 *
 *   num_blocks  number of physical blocks in k_cache and v_cache (both
 *               [num_blocks, block_size, Hkv, d]); 1 <= num_blocks < 2^27.
 *   All other arguments, the result and the errors as paged_attn_decode;
 *   ATTN_ERR_INVALID_ARG also for num_blocks <= 0 when B > 0.
 *
 *   An entry outside [0, num_blocks) among the entries a sequence reads
 *   (j < ceil(seq_len / block_size)) is never dereferenced: its
 *   block_size positions are left out of the softmax, as if masked, and
 *   ATTN_DEVSTATUS_BAD_BLOCK is set.  A query whose every position is left
 *   out gets O = 0.  The pool views the kernels load through end at
 *   num_blocks as well, so no load reaches past the pool.
 */
int paged_attn_decode_checked(const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_table, const int32_t* seq_lens,
                              int B, int Hq, int Hkv, int d, int block_size, int max_blocks,
                              int num_blocks, int num_splits, void* o, attn_stream_t stream);

/*
 * paged_attn_decode_partial - the decode over part of each sequence's keys,
 * returned in a form that other parts can be merged with.
 *
 * Context-parallel decode of long sequences: each device holds a contiguous
 * range of every sequence's cached tokens in its own pool, with its own
 * block table and lengths, and attends the query to that range only.  The
 * per-range results are then merged (attn_lse_merge) after an exchange.  The
 * split rests on the online-softmax statistics of the page "Snelle
 * attention-kernels en operatorfusie versnellen AI-modellen" (the-ai.news),
 * section "FlashAttention-type aandacht en gepagineerde aandacht": keys can
 * be processed in any grouping as long as each group carries its maximum and
 * sum; the natural-log LSE below carries both.
 *
 *   q, k_cache, v_cache, block_table, seq_lens, B, Hq, Hkv, d, block_size,
 *   max_blocks, num_blocks, num_splits: as paged_attn_decode_checked, for
 *                the keys this call sees (seq_lens[b] = the tokens of
 *                sequence b held here; 0 allowed).
 *   o_part       [B, Hq, d] fp32 (written): softmax-weighted average of the
 *                values over the keys seen here, normalised by their own sum.
 *   lse_part     [B, Hq] fp32 (written): ln sum_j exp(scale * <q, k_j>) over
 *                those keys.  A query that sees no key gets o_part = 0 and
 *                lse_part = -inf.
 *
 *   With every key of a sequence in one call, o_part equals the output of
 *   paged_attn_decode before its rounding to bf16.
 *   Supported and errors: as paged_attn_decode_checked; o_part 16-byte and
 *   lse_part 4-byte aligned; ATTN_ERR_INVALID_ARG for a null o_part or
 *   lse_part.  Workspace: as paged_attn_decode when num_splits resolves to
 *   more than 1, none otherwise.
 */
int paged_attn_decode_partial(const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_table, const int32_t* seq_lens,
                              int B, int Hq, int Hkv, int d, int block_size, int max_blocks,
                              int num_blocks, int num_splits, float* o_part, float* lse_part,
                              attn_stream_t stream);

/*
 * attn_lse_merge - merge R partial decode results of the same queries into
 * the final output.
 *
 *   o_parts    [R, B, Hq, d] fp32, lse_parts [R, B, Hq] fp32: R results of
 *              paged_attn_decode_partial over disjoint key ranges (for
 *              instance one per device, gathered over NCCL).
 *   o          [B, Hq, d] bf16 (written):
 *                M = max_r lse_r,  w_r = exp(lse_r - M),
 *                o = sum_r w_r o_r / sum_r w_r,
 *              o = 0 where every lse_r is -inf.  This is the softmax over
 *              the union of the key ranges, since sum_r w_r e^M is the sum
 *              of exp of every score.  The result is deterministic (fixed
 *              order, no atomics).
 *
 *   Supported: d in {64, 128}; 1 <= R <= 65535; o_parts and o 16-byte,
 *   lse_parts 4-byte aligned; sm_100 device.  B == 0 is a no-op.
 *   Errors: ATTN_ERR_INVALID_ARG for R <= 0, B < 0, Hq <= 0, d <= 0 or a
 *   null pointer; ATTN_ERR_UNSUPPORTED otherwise outside the supported set;
 *   ATTN_ERR_CUDA for a launch failure.  No workspace.
 */
int attn_lse_merge(const float* o_parts, const float* lse_parts, int R, int B, int Hq, int d, void* o,
                   attn_stream_t stream);

/*
 * attn_check_support - initialisation-time compatibility check of `device`,
 * in the spirit of the backend check at start-up described in the same
 * section of the page (an incompatible backend is reported as an error at
 * initialisation instead of failing later).  Returns ATTN_OK when the device
 * is an sm_100 part this library was built for, ATTN_ERR_UNSUPPORTED when it
 * is not, ATTN_ERR_CUDA when the device cannot be queried.
 */
int attn_check_support(int device);

/* Static, human-readable name of a status code (never NULL). */
const char* attn_status_string(int status);

/*
 * attn_read_device_status - copy the device status word of the current
 * device into *out (synchronous: waits for the device) and clear it when
 * `clear` != 0.  Bit ATTN_DEVSTATUS_TIMEOUT means a bounded wait inside a
 * kernel gave up.  Returns ATTN_OK or ATTN_ERR_CUDA / ATTN_ERR_INVALID_ARG.
 */
int attn_read_device_status(int* out, int clear);

/*
 * attn_selftest_bounded_wait - exercise the give-up path of the kernels'
 * bounded waits.  Launches one CTA on `stream` that waits, with the same
 * wait routine and the same time limit (about 1 s) as the attention kernels,
 * on an mbarrier that nothing ever arrives on.  The wait gives up, sets
 * ATTN_DEVSTATUS_TIMEOUT in the device status word and the kernel exits; the
 * CUDA context stays usable.  Read the result with attn_read_device_status().
 * Returns ATTN_OK when the launch succeeded.
 */
int attn_selftest_bounded_wait(attn_stream_t stream);

/*
 * paged_attn_prefill - chunked prefill against the paged KV cache: several
 * new query tokens per sequence attend to that sequence's paged context
 * (the paged cache and its block-table translation of the page "Snelle
 * attention-kernels en operatorfusie versnellen AI-modellen", section
 * "FlashAttention-type aandacht en gepagineerde aandacht", combined with the
 * blockwise prefill of attn_fwd).
 *
 *   q            [total_q, Hq, d] bf16: the new tokens of the B sequences,
 *                back to back (rows cu_seqlens_q[b] .. cu_seqlens_q[b+1])
 *   k_cache, v_cache, block_table: as paged_attn_decode
 *   seq_lens     [B] int32: tokens in the cache for sequence b, the new
 *                tokens included (they are the last T_b of them)
 *   cu_seqlens_q [B + 1] int32 prefix sums of the query counts T_b
 *   o            [total_q, Hq, d] bf16 (written); lse [Hq, total_q] fp32 or NULL
 *
 *   Query row i of sequence b sits at position seq_lens[b] - T_b + i; with
 *   causal != 0 it sees the keys at positions <= its own (bottom-right
 *   alignment of attn_fwd with T = T_b, S = seq_lens[b]); otherwise all
 *   seq_lens[b] keys.  Pool slots past the sequence end may hold anything.
 *   max_seqlen_q must be >= every T_b.  seq_lens and block ids are checked
 *   as in paged_attn_decode.
 *   Supported: d in {64, 128}; block_size == 16; Hq % Hkv == 0;
 *   max_blocks < 2^27; sm_100.
 *   Errors: as paged_attn_decode.
 */
int paged_attn_prefill(const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_table, const int32_t* seq_lens, const int32_t* cu_seqlens_q,
                       int B, int Hq, int Hkv, int d, int block_size, int max_blocks,
                       int max_seqlen_q, int total_q, int causal, float scale,
                       void* o, float* lse, attn_stream_t stream);

/*
 * paged_attn_prefill_checked - paged_attn_prefill for a pool of known size
 * num_blocks (1 <= num_blocks < 2^27), with the block-id check of
 * paged_attn_decode_checked: an entry outside [0, num_blocks) is never
 * dereferenced, its positions are masked for every query row and
 * ATTN_DEVSTATUS_BAD_BLOCK is set.  A row that sees no position gets O = 0
 * and LSE = -inf.  Other arguments, results and errors as
 * paged_attn_prefill.
 */
int paged_attn_prefill_checked(const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_table, const int32_t* seq_lens, const int32_t* cu_seqlens_q,
                               int B, int Hq, int Hkv, int d, int block_size, int max_blocks, int num_blocks,
                               int max_seqlen_q, int total_q, int causal, float scale,
                               void* o, float* lse, attn_stream_t stream);

/*
 * paged_attn_decode_fp8 - paged_attn_decode with the KV cache stored as FP8
 * e4m3 (OCP e4m3fn: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits),
 * one scale per tensor: K = k_scale * k_cache, V = v_scale * v_cache.  Half
 * the bytes per cached token of the bf16 cache.
 *
 *   k_cache, v_cache [num_blocks, block_size, Hkv, d] e4m3 bytes (16-byte
 *   aligned); all other arguments and the result as paged_attn_decode.
 *   The arithmetic is f16 x f16 -> fp32 on the tensor cores (e4m3 values are
 *   exact in f16; q and P are rounded to f16).
 *   Supported: d == 128; block_size == 16; 1 <= Hq/Hkv <= 8; sm_100.
 *   Errors: as paged_attn_decode; ATTN_ERR_INVALID_ARG also for a scale that
 *   is not finite and positive.
 */
int paged_attn_decode_fp8(const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* block_table, const int32_t* seq_lens,
                          int B, int Hq, int Hkv, int d, int block_size, int max_blocks,
                          int num_splits, float k_scale, float v_scale, void* o, attn_stream_t stream);

/*
 * paged_attn_decode_fp8_checked - paged_attn_decode_fp8 for a pool of known
 * size num_blocks, with the block-id check of paged_attn_decode_checked.
 */
int paged_attn_decode_fp8_checked(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* block_table, const int32_t* seq_lens,
                                  int B, int Hq, int Hkv, int d, int block_size, int max_blocks,
                                  int num_blocks, int num_splits, float k_scale, float v_scale, void* o,
                                  attn_stream_t stream);

/*
 * paged_attn_decode_noalloc - paged_attn_decode for callers that must not
 * allocate device memory during the call.
 *
 * The pages describe no such variant; it exists for integration only.  Some
 * callers cannot let a library call cudaMalloc or draw from a memory pool:
 * code running inside a pre-planned memory budget (an inference server that
 * has already handed all free memory to its KV-cache pool), allocators that
 * must not be re-entered from a callback, or callers that forbid any
 * allocation on their hot path.  This entry point takes the same arguments
 * and computes the same result as paged_attn_decode, but its split-KV
 * partials live in one fixed scratch array compiled into the library
 * (ATTN_NOALLOC_SCRATCH_BYTES per GPU, held by every GPU that loads the
 * library until the process exits).  It calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *
 *   Limit: num_splits * B * Hq * (d + 1) * 4 bytes of partials must not
 *   exceed ATTN_NOALLOC_SCRATCH_BYTES.  With num_splits <= 0 the automatic
 *   split count is lowered until its partials fit (down to one split, which
 *   uses no scratch), so an automatic call never fails on this limit; an
 *   explicit num_splits whose partials do not fit returns
 *   ATTN_ERR_UNSUPPORTED before anything is launched.
 *   First call on a device: it looks up the scratch array's device address
 *   (cudaGetSymbolAddress, with that device current) and sets the kernels'
 *   shared-memory limits; make that first call before any stream capture.
 *   Sharing: every call on a device uses the same scratch array and it keeps
 *   the previous call's contents (no part of it needs to start at zero: each
 *   partial the merge reads is written earlier in the same call).  Calls that
 *   can overlap on the GPU (different streams without ordering between them)
 *   race on the scratch and give undefined results; serialise them.
 *   seq_lens and block ids are checked as in paged_attn_decode.
 *   Errors: as paged_attn_decode, plus the limit above.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (16u << 20)

int paged_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_table, const int32_t* seq_lens,
                              int B, int Hq, int Hkv, int d, int block_size, int max_blocks,
                              int num_splits, void* o, attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
