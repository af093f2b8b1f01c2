/*
 * attn_gqa.h -- exact tiled grouped-query attention for NVIDIA B200 (sm_100a).
 *
 * The operation (both calls):
 *
 *   O = softmax(scale * Q K^T + mask) V
 *
 * computed exactly -- no approximation -- tile by tile with an online softmax
 * that keeps only a running row maximum and row sum, so the Lq x Lk score
 * table never reaches device memory.  This is the construction the page
 * "어텐션 구현 고르기, SDPA·FlashAttention 메모리와 GPU 비용" (SDPA / FlashAttention
 * selection guide) describes in its section on eager-attention memory: the
 * score table is cut into on-chip blocks and only a max and a sum per row
 * survive, memory grows linearly in length, and the result is the same as the
 * eager computation up to the order of floating-point sums.
 *
 * Grouped-query heads: G = Hq / Hkv consecutive query heads share one key /
 * value head; query head h reads KV head h / G.  G = 1 is multi-head and
 * Hkv = 1 is multi-query attention (NVIDIA attention-optimisation page,
 * "Parameter one: group size").
 *
 * Conventions shared by every call:
 *   - Tensors are dense, row-major, and live in device memory owned by the
 *     caller.  The library never frees or keeps a pointer after a call
 *     returns (the kernels it launched may still be reading them: the
 *     caller keeps them alive until `stream` has passed the work).
 *   - bf16 tensors are passed as `const void*` / `void*` to 16-bit bfloat16
 *     elements.  Base addresses must be 16-byte aligned.
 *   - LSE is the natural-log log-sum-exp of the scaled, masked scores of a
 *     row: LSE_i = m_i + ln(sum_j exp(scale * q_i.k_j - m_i)).  A row that
 *     sees no key gets O = 0 and LSE = -inf.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work on it; none synchronises the host.  A call that
 *     launches two kernels (a split kernel and the combine or merge of its
 *     partial results) launches the second as a programmatic dependent of the
 *     first: it may be scheduled while the first is finishing but reads
 *     nothing before the first has completed, so stream order, events and
 *     graph capture see the call as one piece of work.
 *   - Return value: ATTN_OK, or a negative attn_status_t.  Argument checks
 *     happen before anything is enqueued, so a failed call has no effect.
 *     attn_last_error() gives a one-line description of the last failure on
 *     the calling thread.
 *   - Per-device state: on first use of a device the library looks up, and
 *     then keeps for the life of the process, the addresses of its own device
 *     arrays, kernel attributes, and (attn_prefill_host) two streams and a few
 *     events.  All of these belong to the device's primary context, so the
 *     library must not be called again after that context is destroyed
 *     (cudaDeviceReset, or a reset of the primary context through the driver).
 */
#ifndef ATTN_GQA_H
#define ATTN_GQA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = -1, /* null pointer, bad size, Hq % Hkv != 0, bad scale, misalignment */
    ATTN_ERR_UNSUPPORTED = -2, /* valid but not built: D not in {64, 128, 256}, group size too large */
    ATTN_ERR_WORKSPACE = -3,   /* decode workspace missing or smaller than required */
    ATTN_ERR_CUDA = -4         /* a CUDA runtime call or kernel launch failed */
} attn_status_t;

/*
 * attn_prefill -- causal (or full) attention of Lq query rows against Lk keys.
 *
 * Defined by the SDPA / FlashAttention selection guide: the eager
 * computation in "eager attention memory", its tiled equivalent in the same
 * section, and the mask alignment of "is_causal mask alignment, the trap
 * with a KV cache".  With is_causal != 0 the mask is aligned bottom-right:
 * query row i (0-based) sees key j iff j <= i + (Lk - Lq).  For Lq == Lk this
 * is the usual lower triangle; for Lq < Lk (a chunk of new tokens appended to
 * Lk - Lq cached ones) the rows are the last Lq positions of the sequence.
 * With is_causal == 0 every row sees all Lk keys.
 *
 *   q    [B, Hq,  Lq, D]  bf16, read
 *   k    [B, Hkv, Lk, D]  bf16, read
 *   v    [B, Hkv, Lk, D]  bf16, read
 *   out  [B, Hq,  Lq, D]  bf16, written
 *   lse  [B, Hq,  Lq]     fp32, written; may be NULL (not written)
 *   scale: finite and > 0 (usually 1/sqrt(D))
 *   D: 64, 128 or 256 (the head dims the NVIDIA attention page recommends,
 *   "Parameter two: head dimension", plus 64).  G = Hq / Hkv: 1 .. 128.
 *   B == 0 or Lq == 0: nothing to do, returns ATTN_OK.
 *   Lk == 0: every row sees no key (O = 0, LSE = -inf).
 *
 * q and out may be NULL only when they are empty (B == 0 or Lq == 0), k and
 * v only when they are empty (B == 0 or Lk == 0).
 *
 * Errors: ATTN_ERR_INVALID_ARG for a null non-empty tensor, negative sizes, Hq or
 * Hkv < 1, Hq % Hkv != 0, non-finite or non-positive scale, or a base
 * address not 16-byte aligned; ATTN_ERR_UNSUPPORTED for D outside {64, 128, 256}
 * or G > 128; ATTN_ERR_CUDA when a launch fails.
 *
 * Concurrency: for D = 64 and 128 the kernel is persistent and hands out its
 * work from a pair of counters in the library's device memory.  An ordinary
 * call takes the next of 256 such pairs in turn; a call made while `stream` is
 * being captured into a CUDA graph takes the next of 1024 further pairs, which
 * that graph then uses on every replay, so graph replays and ordinary calls
 * never share counters.  The rules that follow:
 *   - ordinary calls on one stream may follow each other without limit; at
 *     most 256 ordinary calls may be in flight at the same time across streams;
 *   - a graph holding this call must not be replayed while it is still
 *     running (e.g. on two streams at once), and two graphs whose captures of
 *     this call lie a multiple of 1024 captures apart must not run at the
 *     same time.
 * A launch that finds its counters used by another launch at the same time
 * sets ATTN_DEVERR_SCHED in the device error word (its results may then be
 * incomplete).
 */
int attn_prefill(const void* q, const void* k, const void* v, void* out, float* lse,
                 int B, int Hq, int Hkv, int Lq, int Lk, int D, float scale, int is_causal,
                 void* stream);

/*
 * attn_prefill_workspace_size / attn_prefill_ws -- attn_prefill with a
 * workspace it may use to even out the end of a launch.
 *
 * Same operation, arguments, layouts, limits and results as attn_prefill (the
 * guide's eager computation, tiled), plus:
 *   workspace   device memory of attn_prefill_workspace_size(...) bytes,
 *               256-byte aligned, owned by the caller; may be NULL when that
 *               size is 0
 * A launch of D <= 128 takes its work units (a KV group, 2 x 128 query rows)
 * one wave per SM at a time.  When every query of the launch sees most keys
 * (chunked prefill, Lq much smaller than Lk) the units are nearly equal, and a
 * unit count between 1 and 4 waves that is not a multiple of the SM count ends
 * in a part-filled wave.  attn_prefill_ws then cuts the units of that last
 * wave into 4 runs of key tiles, writes their normalised fp32 partial results
 * and log-sum-exps to the workspace and merges them (the single-device form of
 * the split over keys of the NVIDIA attention page, "Parameter four:
 * parallelism").  The result is the same attention up to the rounding of the
 * merge.  attn_prefill_workspace_size returns 0 when no such split applies
 * (then attn_prefill_ws is attn_prefill); it depends on the sizes and on the
 * current device's SM count.  Errors: as attn_prefill, plus ATTN_ERR_WORKSPACE
 * for a workspace smaller than required and ATTN_ERR_INVALID_ARG for a
 * misaligned one.
 */
size_t attn_prefill_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int D, int is_causal);
int attn_prefill_ws(const void* q, const void* k, const void* v, void* out, float* lse,
                    int B, int Hq, int Hkv, int Lq, int Lk, int D, float scale, int is_causal,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_prefill_host_scratch_size / attn_prefill_host -- attn_prefill with
 * q, k, v, out and lse in HOST memory: the call copies the inputs to the device,
 * computes, and copies the results back, overlapping the three.
 *
 * Same operation, arguments, layouts and limits as attn_prefill, except:
 *   q, k, v, out, lse  host pointers (page-locked memory lets the copies run
 *                      asynchronously and overlap; pageable memory works but
 *                      each copy then waits for the host); lse may be NULL
 *   scratch            device memory of attn_prefill_host_scratch_size(...)
 *                      bytes, 256-byte aligned, owned by the caller (two
 *                      slots of one work unit each; see below)
 *
 * The work is cut into units of one sequence and a run of KV heads (the
 * smallest divisor of Hkv whose kernel still fills a wave of CTAs); for each
 * unit the q, k, v slabs are copied in on a library-owned stream, the prefill
 * kernel runs on `stream`, and the out and lse slabs are copied back on a second
 * library-owned stream, with events ordering the two device slots, so one
 * unit's copy in, the previous unit's kernel and the one before's copy out run
 * at once.  The library creates its two copy streams and a few events once per
 * device and keeps them for the life of the process.
 *
 * Completion: when `stream` has passed the work this call enqueued, every
 * result is in host memory.  The host buffers must stay valid until then.
 * Calls from several host threads on one device are serialised while they
 * enqueue.  Errors: as attn_prefill, plus ATTN_ERR_WORKSPACE for a missing or
 * small scratch and ATTN_ERR_INVALID_ARG for a misaligned one; a CUDA failure
 * part-way returns ATTN_ERR_CUDA with the units before it enqueued.
 */
size_t attn_prefill_host_scratch_size(int B, int Hq, int Hkv, int Lq, int Lk, int D);
int attn_prefill_host(const void* q, const void* k, const void* v, void* out, float* lse,
                      int B, int Hq, int Hkv, int Lq, int Lk, int D, float scale, int is_causal,
                      void* scratch, size_t scratch_bytes, void* stream);

/*
 * attn_decode_workspace_size -- bytes of scratch attn_decode needs for these
 * sizes (split-KV partial outputs and their log-sum-exps).  Depends only on
 * the arguments.  Returns 0 for sizes attn_decode would reject.
 */
size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int D);

/*
 * attn_decode -- one new query token per sequence against a KV cache.
 *
 * Defined by the same guide's "use_cache" section and the is_causal section:
 * cached keys and values of earlier tokens do not change, and the single new
 * query row sees every cached key, so no mask is needed.  Sequence b has
 * seqlens[b] valid cache rows, 0 .. seqlens[b]-1; rows at or beyond
 * seqlens[b] are never used (they may hold anything, NaN included).
 *
 * The cache is split along its length; each piece is reduced with its own
 * online softmax and the pieces are merged by their log-sum-exps (the
 * single-GPU form of the KV parallelism on the NVIDIA attention page,
 * "Parameter four: parallelism").
 *
 *   q        [B, Hq, D]          bf16, read
 *   k_cache  [B, Hkv, Lmax, D]   bf16, read
 *   v_cache  [B, Hkv, Lmax, D]   bf16, read
 *   seqlens  [B]                 int32 in device memory, each in [0, Lmax];
 *                                a value outside is clamped into range and
 *                                flags ATTN_DEVERR_SEQLEN (attn_device_error)
 *   out      [B, Hq, D]          bf16, written
 *   lse      [B, Hq]             fp32, written; may be NULL
 *   workspace: device memory of at least attn_decode_workspace_size(...)
 *              bytes, 256-byte aligned, owned by the caller; its contents on
 *              entry do not matter and on return are unspecified.  Two calls
 *              in flight at once must not share one workspace.
 *   D: 64, 128 or 256.  G = Hq / Hkv: 1 .. 128.  B == 0 returns ATTN_OK.
 *
 * Errors: as attn_prefill, plus ATTN_ERR_WORKSPACE for a null or too small
 * workspace.
 */
int attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                void* out, float* lse, int B, int Hq, int Hkv, int Lmax, int D, float scale,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_decode_host_workspace_size / attn_decode_host -- attn_decode for a
 * caller whose new query rows arrive in, and whose results go back to, HOST
 * memory, while the KV cache stays resident on the device (a cache is device
 * state that decode steps append to; the "use_cache" section of the SDPA
 * guide).  One call copies q and seqlens in, decodes, and copies out and lse
 * back, all enqueued on `stream` in that order.
 *
 *   q        [B, Hq, D]          bf16, HOST memory, read
 *   k_cache  [B, Hkv, Lmax, D]   bf16, device memory, read (as attn_decode)
 *   v_cache  [B, Hkv, Lmax, D]   bf16, device memory, read
 *   seqlens  [B]                 int32, HOST memory, read (values as attn_decode)
 *   out      [B, Hq, D]          bf16, HOST memory, written
 *   lse      [B, Hq]             fp32, HOST memory, written; may be NULL
 *   workspace device memory of attn_decode_host_workspace_size(...) bytes,
 *            256-byte aligned, owned by the caller: attn_decode's split
 *            partials followed by device copies of q, out, lse and seqlens
 *
 * Page-locked host buffers let the copies run asynchronously; with pageable
 * memory each copy waits for the host.  Completion: when `stream` has passed
 * the work this call enqueued, out and lse hold the results; the host buffers
 * must stay valid until then.  Errors: as attn_decode (checked before anything
 * is enqueued), ATTN_ERR_WORKSPACE for a missing or small workspace,
 * ATTN_ERR_INVALID_ARG for a misaligned one, ATTN_ERR_CUDA if a copy cannot
 * be enqueued.  attn_decode_host_workspace_size returns 0 for sizes
 * attn_decode would reject and for B == 0.
 */
size_t attn_decode_host_workspace_size(int B, int Hq, int Hkv, int Lmax, int D);
int attn_decode_host(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                     void* out, float* lse, int B, int Hq, int Hkv, int Lmax, int D, float scale,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_decode_partial / attn_decode_merge -- decode split across devices by
 * cache rows (the KV parallelism of the NVIDIA attention page, "Parameter
 * four: parallelism"): each device holds a disjoint set of every sequence's
 * cached rows, computes attention over its own rows with attn_decode_partial,
 * the partial results are exchanged (an all-gather), and attn_decode_merge
 * combines them into exactly the attention over all rows.
 *
 * attn_decode_partial: attn_decode (same arguments, layouts, limits, workspace
 * from attn_decode_workspace_size and errors) with its results left unrounded
 * for the merge:
 *   o_part    [B, Hq, D] fp32, written: O over this caller's rows
 *   lse_part  [B, Hq]    fp32, written: natural-log LSE over those rows (-inf
 *             when a sequence has none here); must not be NULL
 *
 * attn_decode_merge:
 *   o_parts   [n_parts, rows, D] fp32, read (rows = B * Hq for decode)
 *   lse_parts [n_parts, rows] fp32, read
 *   out       [rows, D] bf16, written: sum_p exp(lse_p - lse) o_p
 *   lse       [rows] fp32 or NULL, written: ln sum_p exp(lse_p)
 *   n_parts >= 1; D 64, 128 or 256; o_parts and out 16-byte aligned.
 * A row with no rows in any part gets O = 0 and LSE = -inf.  Errors:
 * ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED (D), ATTN_ERR_CUDA.  rows == 0
 * returns ATTN_OK.
 */
int attn_decode_partial(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                        float* o_part, float* lse_part, int B, int Hq, int Hkv, int Lmax, int D, float scale,
                        void* workspace, size_t workspace_bytes, void* stream);
int attn_decode_merge(const float* o_parts, const float* lse_parts, int n_parts, int rows, int D,
                      void* out, float* lse, void* stream);

/*
 * attn_kvp_signal / attn_kvp_wait / attn_decode_merge_peers -- the same KV
 * parallelism with the exchange fused into the merge: each device leaves its
 * attn_decode_partial results in its own memory, and the merge on every device
 * reads all parts where they lie -- its own memory or a peer's, over NVLink,
 * with plain loads -- instead of all-gathering them first.  Epoch flags order
 * the steps; an epoch is a 32-bit counter that grows by one per step, and a
 * flag "has reached" a value when (int32_t)(flag - value) >= 0.
 *
 * One step, epoch e, on device r of n (ready and consumed are n-entry uint32
 * arrays in device r's memory, zero before the first step):
 *   1. attn_kvp_wait(consumed, n, e - 1)   (steps after the first) -- every
 *      device has finished reading this device's previous parts
 *   2. attn_decode_partial into this device's part buffers
 *   3. attn_kvp_signal({&ready_on_device_p[r] for p < n}, n, e)
 *   4. attn_decode_merge_peers(o_ptrs, lse_ptrs, ready, e, n, ...)
 *   5. attn_kvp_signal({&consumed_on_device_p[r] for p < n}, n, e)
 * all on one stream.  Every pointer must be valid in the calling process
 * (peer memory mapped into it, e.g. through CUDA IPC or symmetric memory).
 *
 * attn_kvp_signal: after everything enqueued before it on `stream` is visible
 *   system-wide, stores `value` to *flag_ptrs[i] (i < n) with release
 *   semantics.  flag_ptrs: device array of n device pointers.
 * attn_kvp_wait: makes `stream` wait until flags[0 .. n) (device array) have
 *   all reached `value`.
 * attn_decode_merge_peers: attn_decode_merge with part p's O at o_ptrs[p]
 *   ([rows, D] fp32) and its LSE at lse_ptrs[p] ([rows] fp32, natural log),
 *   device arrays of n_parts pointers; each CTA first waits until ready[0 ..
 *   n_parts) have reached `value`.  out [rows, D] bf16 16-byte aligned, lse
 *   [rows] fp32 or NULL.
 * Every wait gives up after about 2 s, sets ATTN_DEVERR_TIMEOUT and lets the
 * kernel end (the merge then leaves out and lse unwritten).  Errors:
 * ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED (D), ATTN_ERR_CUDA; n == 0 or
 * rows == 0 returns ATTN_OK.
 */
int attn_kvp_signal(unsigned int* const* flag_ptrs, int n, unsigned int value, void* stream);
int attn_kvp_wait(const unsigned int* flags, int n, unsigned int value, void* stream);
int attn_decode_merge_peers(const float* const* o_ptrs, const float* const* lse_ptrs, const unsigned int* ready,
                            unsigned int value, int n_parts, int rows, int D, void* out, float* lse, void* stream);

/*
 * attn_decode_mq_workspace_size -- bytes of scratch attn_decode_mq needs for
 * these sizes.  Depends only on the arguments; 0 for sizes it would reject.
 */
size_t attn_decode_mq_workspace_size(int B, int Hq, int Hkv, int Lq, int Lmax, int D);

/*
 * attn_decode_mq -- Lq >= 1 new tokens per sequence against a KV cache: the
 * verify step of speculative decoding, or a small chunk of new tokens.
 *
 * The SDPA / FlashAttention selection guide's is_causal section works this
 * case out for two queries (its L = 2 rows: "the verify step of speculative
 * decoding or chunked prefill"): the new tokens' K/V are already the last Lq
 * rows of the cache, and the mask must be aligned bottom-right.  So with
 * n = seqlens[b], new token i (0-based) of sequence b sees cache rows
 * 0 .. n - Lq + i; a token that sees no row (n < Lq - i) gets O = 0 and
 * LSE = -inf.  Lq = 1 is exactly attn_decode.
 *
 *   q        [B, Hq, Lq, D]      bf16, read
 *   k_cache, v_cache, seqlens    as attn_decode (rows >= seqlens[b] unused)
 *   out      [B, Hq, Lq, D]      bf16, written
 *   lse      [B, Hq, Lq]         fp32, written; may be NULL
 *   workspace: at least attn_decode_mq_workspace_size(...) bytes, as attn_decode
 *   D: 64, 128 or 256.  G * Lq <= 128 (G = Hq / Hkv).
 *
 * Errors: as attn_decode, plus ATTN_ERR_INVALID_ARG for Lq < 1 and
 * ATTN_ERR_UNSUPPORTED for G * Lq > 128.
 */
int attn_decode_mq(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                   void* out, float* lse, int B, int Hq, int Hkv, int Lq, int Lmax, int D, float scale,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_decode_paged_workspace_size -- bytes of scratch attn_decode_paged needs;
 * 0 for sizes it would reject.
 */
size_t attn_decode_paged_workspace_size(int B, int Hq, int Hkv, int Lq, int page_size, int max_pages, int D);

/*
 * attn_decode_paged -- attn_decode_mq over a paged KV cache: the cache lives
 * in fixed-size pages of a shared pool, and a block table says which pages
 * hold each sequence (the layout serving engines use so that sequences can
 * grow without copying).  The arithmetic is that of attn_decode_mq; only
 * where cache row r of sequence b is read from changes:
 *
 *   row r of sequence b, KV head g  =  k_pages[block_table[b][r / page_size], g, r % page_size, :]
 *
 *   q            [B, Hq, Lq, D]                  bf16, read
 *   k_pages      [n_pages, Hkv, page_size, D]    bf16, read (pages not in use may hold anything)
 *   v_pages      [n_pages, Hkv, page_size, D]    bf16, read
 *   block_table  [B, max_pages]                  int32 in device memory; entries for the pages
 *                                                a sequence uses must lie in [0, n_pages); one
 *                                                outside is replaced by page 0 and flags
 *                                                ATTN_DEVERR_PAGE
 *   seqlens      [B]                             int32 in device memory, each in
 *                                                [0, page_size * max_pages]
 *   out          [B, Hq, Lq, D] bf16;  lse [B, Hq, Lq] fp32 or NULL
 *   page_size: a positive multiple of 64.  D: 64, 128 or 256.  G * Lq <= 128.
 *
 * Errors: as attn_decode_mq, plus ATTN_ERR_INVALID_ARG for a page_size that
 * is not a positive multiple of 64, n_pages or max_pages < 1, or a null
 * block_table.
 */
int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                      const int32_t* seqlens, void* out, float* lse, int B, int Hq, int Hkv, int Lq, int n_pages,
                      int page_size, int max_pages, int D, float scale, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * attn_decode_noalloc -- attn_decode for callers that cannot allocate device
 * memory: the split partials live in a scratch array that the library itself
 * declares at file scope (ATTN_DECODE_NOALLOC_SCRATCH_BYTES per GPU, reserved
 * on every GPU that loads the library and held until the process exits).
 *
 * The pages have no counterpart to this call; it exists for callers whose
 * device memory is all owned by someone else -- an inference engine that
 * reserves nearly all of HBM for its own pool up front, or a caller that must
 * not call cudaMalloc on its hot path because cudaMalloc can synchronise the
 * device and stall every stream -- and who therefore cannot hand attn_decode
 * a workspace.
 *
 * Arguments, layouts and results are those of attn_decode, without the
 * workspace.  Nothing is allocated: no cudaMalloc, cudaFree or allocating
 * library routine is called.
 *   - Sizes whose partials need more than ATTN_DECODE_NOALLOC_SCRATCH_BYTES
 *     (attn_decode_workspace_size(...) > the limit) are rejected with
 *     ATTN_ERR_WORKSPACE; attn_decode with a caller workspace has no limit.
 *   - The first call on a device looks up the scratch array's device address
 *     (once per device, with that device current); make that first call
 *     before any stream capture.
 *   - Every call on a device shares the one scratch array, which keeps the
 *     previous call's contents.  Nothing in it has to start at zero: each
 *     call writes every partial it later reads.  Calls whose kernels overlap
 *     on the GPU (different streams, no ordering between them) race on the
 *     array and produce wrong results; order them on one stream or with events.
 */
#define ATTN_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)

int attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlens,
                        void* out, float* lse, int B, int Hq, int Hkv, int Lmax, int D, float scale,
                        void* stream);

/*
 * 8-bit KV cache element formats (attn_decode_kv8).
 *
 * The page "Attention Slack" (llama.cpp serving Gemma 4 on one RTX 3090)
 * runs its server with 8-bit K and V caches (the q8_0 cache type, in its
 * server configuration); the NVIDIA attention page ("Prefill and decode are
 * two different tasks") has decode bound by reading the cache, so one byte
 * per element halves the bytes a token costs.  The pages define neither
 * format; these are the two this library reads:
 *
 *   ATTN_KV_E4M3  OCP FP8 E4M3 codes (1 sign, 4 exponent bits with bias 7,
 *                 3 mantissa bits; exponent 0 is subnormal; no infinities;
 *                 S.1111.111 is NaN; largest finite value 448).  Scales:
 *                 k_scale and v_scale are `const float*` arrays [Hkv] in
 *                 device memory; element = scale[g] * value(code).
 *   ATTN_KV_Q8_0  int8 codes (two's complement), one fp16 scale per 32
 *                 consecutive values of a cache row, as q8_0 blocks are.
 *                 The codes and the scales are two planes (not interleaved
 *                 34-byte blocks) so both are TMA-aligned: k_scale and
 *                 v_scale point to fp16 arrays [B, Hkv, Lmax, D / 32];
 *                 element [b, g, r, d] = scale[b, g, r, d / 32] * code.
 */
#define ATTN_KV_E4M3 1
#define ATTN_KV_Q8_0 2

/*
 * attn_decode_kv8_workspace_size -- bytes of scratch attn_decode_kv8 needs
 * for these sizes.  Returns 0 for sizes attn_decode_kv8 would reject or B == 0.
 */
size_t attn_decode_kv8_workspace_size(int B, int Hq, int Hkv, int Lq, int Lmax, int D);

/*
 * attn_decode_kv8 -- attn_decode_mq (Lq >= 1 new query rows per sequence,
 * bottom-right against the cache) with an 8-bit K/V cache.
 *
 * The result is the exact attention over the dequantised cache: with K and V
 * replaced by their element values (above), the same O and LSE as
 * attn_decode_mq.  The MMAs run in f16 with fp32 sums: every E4M3 value and
 * every int8 value is exact in f16, Q is brought into f16 range by a power of
 * two per row (exact), and P is rounded to f16.
 *
 *   q          [B, Hq, Lq, D]     bf16, read
 *   k_cache    [B, Hkv, Lmax, D]  8-bit codes (uint8 storage), read; rows at
 *   v_cache    [B, Hkv, Lmax, D]  or past seqlens[b] are never used (NaN
 *                                 codes there have no effect)
 *   k_scale, v_scale              per kv_format (above), read
 *   kv_format  ATTN_KV_E4M3 or ATTN_KV_Q8_0
 *   seqlens    [B] int32, read; 0 <= seqlens[b] <= Lmax
 *   out        [B, Hq, Lq, D] bf16, written;  lse [B, Hq, Lq] fp32 or NULL
 *   workspace  attn_decode_kv8_workspace_size(...) bytes, 256-byte aligned
 *   D: 64 or 128.  G * Lq <= 64.  ATTN_KV_Q8_0 needs Lmax % 4 == 0 and
 *   16-byte aligned scale planes; ATTN_KV_E4M3 4-byte aligned scale arrays.
 *
 * Errors: ATTN_ERR_INVALID_ARG (null or misaligned pointers, unknown
 * kv_format, Lq < 1, Lmax < 1, Q8_0 with Lmax % 4 != 0, Hq % Hkv != 0, bad
 * scale), ATTN_ERR_UNSUPPORTED (D not 64 or 128, G * Lq > 64),
 * ATTN_ERR_WORKSPACE, ATTN_ERR_CUDA.  B == 0 returns ATTN_OK.
 */
int attn_decode_kv8(const void* q, const void* k_cache, const void* v_cache, const void* k_scale,
                    const void* v_scale, int kv_format, const int32_t* seqlens, void* out, float* lse,
                    int B, int Hq, int Hkv, int Lq, int Lmax, int D, float scale, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * attn_decode_kv8_paged_workspace_size / attn_decode_kv8_paged -- attn_decode_kv8
 * over a paged 8-bit cache: the page layout of attn_decode_paged (pools
 * [n_pages, Hkv, page_size, D], block_table [B, max_pages], logical row r of
 * sequence b in page block_table[b][r / page_size] at row r % page_size) with
 * 8-bit codes.  ATTN_KV_Q8_0 scale pools are [n_pages, Hkv, page_size, D / 32]
 * fp16, paged like the codes; ATTN_KV_E4M3 scales stay [Hkv] fp32.
 *   page_size: a positive multiple of 64.  Other arguments, limits and
 *   errors as attn_decode_kv8 and attn_decode_paged; block-table entries
 *   outside [0, n_pages) set ATTN_DEVERR_PAGE and are never dereferenced.
 */
size_t attn_decode_kv8_paged_workspace_size(int B, int Hq, int Hkv, int Lq, int page_size, int max_pages, int D);
int attn_decode_kv8_paged(const void* q, const void* k_pages, const void* v_pages, const void* k_scale,
                          const void* v_scale, int kv_format, const int32_t* block_table, const int32_t* seqlens,
                          void* out, float* lse, int B, int Hq, int Hkv, int Lq, int n_pages, int page_size,
                          int max_pages, int D, float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_selftest_kv8_convert -- diagnostic: out[i] = the f16x2 (two f16 bit
 * patterns, code byte 0 in bits 0-15) that attn_decode_kv8 feeds its MMAs for
 * the two 8-bit codes in codes[i] (byte 0 in bits 0-7), for kv_format
 * ATTN_KV_E4M3 (the code's value) or ATTN_KV_Q8_0 (the int8 value, unscaled).
 * Device arrays of n elements; enqueued on `stream`.
 */
int attn_selftest_kv8_convert(const uint16_t* codes, uint32_t* out, int n, int kv_format, void* stream);

/*
 * attn_selftest_wait -- diagnostic: makes the kernels' bounded pipeline wait
 * run out, without touching any real pipeline.  One CTA of two warps: a
 * "producer" announces bytes on a barrier that never arrive (no copy is
 * issued) and then waits, with the kernels' usual ~2 s limit, for the
 * "consumer" to free the entry; the consumer waits on the first barrier with
 * a limit of limit_ns nanoseconds (0 < limit_ns <= 2e9).  The consumer's wait
 * gives up, sets ATTN_DEVERR_TIMEOUT in the device error word and raises the
 * CTA's abort flag, which ends the producer's wait too.
 *   result: device int[4], written: {producer wait succeeded (0/1), producer
 *   wait time in us, consumer wait succeeded (0/1), consumer wait time in us}.
 * Enqueued on `stream`; the caller clears the error word afterwards
 * (attn_device_error with reset).  Errors: ATTN_ERR_INVALID_ARG, ATTN_ERR_CUDA.
 */
int attn_selftest_wait(unsigned long long limit_ns, int* result, void* stream);

/*
 * attn_prefill_sched_busy -- diagnostic: synchronise the current device and
 * count the prefill scheduling counters (see attn_prefill, "Concurrency")
 * that are not zero.  Between launches every counter is zero, also after a
 * launch that gave up on a wait.  Returns ATTN_OK or ATTN_ERR_CUDA /
 * ATTN_ERR_INVALID_ARG.
 */
int attn_prefill_sched_busy(int* busy);

/*
 * attn_prefill_split_plan -- diagnostic, host only (no device call): the
 * key-split plan attn_prefill_ws would use on a device with n_sm SMs.  Writes
 * *n_full (whole work units handed out first) and *n_items (work items of the
 * launch: n_full plus 4 per cut unit; n_items == n_full when nothing is cut;
 * both 0 for head dim 256, whose launches are not persistent, and for invalid
 * arguments) and returns the workspace bytes (attn_prefill_workspace_size on
 * such a device; 0 when nothing is cut).  n_full / n_items may be NULL.
 */
size_t attn_prefill_split_plan(int B, int Hq, int Hkv, int Lq, int Lk, int D, int is_causal, int n_sm,
                               int* n_full, int* n_items);

/* attn_status_string -- a static name for a status code; never NULL. */
const char* attn_status_string(int status);

/* attn_last_error -- description of the last failure on this host thread
 * ("" if none).  The string stays valid until the thread's next call. */
const char* attn_last_error(void);

/*
 * Device-side error word.  Kernels never trap: a wait that runs out of time
 * (a pipeline barrier that never completes) or an out-of-range seqlens value
 * sets a bit here and the kernel returns early.
 */
#define ATTN_DEVERR_TIMEOUT 0x1u  /* a pipeline wait gave up after ~2 s */
#define ATTN_DEVERR_SEQLEN  0x2u  /* a seqlens value was outside [0, Lmax] */
#define ATTN_DEVERR_PAGE    0x4u  /* a block_table entry was outside [0, n_pages) */
#define ATTN_DEVERR_SCHED   0x8u  /* a prefill launch shared its scheduling counters with another
                                     launch running at the same time (see attn_prefill) */
#define ATTN_DEVERR_BOUNDS  0x10u /* only in the library built with -DATTN_DEBUG_BOUNDS=1: a work-unit
                                     mapping, ring position, TMA coordinate or output index fell
                                     outside its tensor (a checking build for tests) */

/*
 * attn_device_error -- synchronise the current device, copy its error word
 * into *flags and, if reset != 0, clear it.  Diagnostic call, not for the hot
 * path.  Returns ATTN_OK or ATTN_ERR_CUDA / ATTN_ERR_INVALID_ARG.
 */
int attn_device_error(unsigned int* flags, int reset);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_GQA_H */
