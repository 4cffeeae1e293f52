/*
 * attn_b200.h -- C ABI of the B200 (sm_100a) exact-attention library.
 *
 * Two operations, both exact scaled-dot-product attention
 *     O = softmax(scale * Q K^T + M) V,   LSE = log sum_j exp(scale * q . k_j)
 * as defined in "Fast Attention Kernels and Operator Fusion" (wpnews.pro),
 * section "FlashAttention-Style Kernels" (the attention equation with an
 * additive mask M; is_causal=True makes M = -inf above the diagonal), fused so
 * that the score matrix never reaches HBM; and its decode form over a paged KV
 * cache read through a block table (same page, section "Paged Attention
 * Kernels").
 *
 * Conventions for every entry point
 *   - bf16 tensors are passed as pointers to raw bfloat16 bits (attn_bf16);
 *     all tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned, contiguous, and must stay valid until the work queued on
 *     `stream` has finished.  The library never frees or retains them.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream) of the current
 *     device.  Calls only enqueue work: they never synchronise, never allocate
 *     device memory, and return before the kernels run.
 *   - The return value is an attn_status.  Argument errors are detected on the
 *     host before anything is enqueued.  There is no fallback path: an
 *     unsupported input is an error, never a slower kernel.  Errors raised
 *     while the kernels run (a broken pipeline wait, a block-table entry
 *     outside the pool) are recorded in a device error word that
 *     attn_device_status() reads.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t attn_bf16; /* raw IEEE bfloat16 bits */

typedef enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_NULL = 1,        /* a required pointer is NULL */
  ATTN_ERR_SHAPE = 2,       /* a size is out of range or inconsistent */
  ATTN_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  ATTN_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required */
  ATTN_ERR_UNSUPPORTED = 5, /* valid input the library has no kernel for */
  ATTN_ERR_LAUNCH = 6,      /* CUDA refused the launch (see attn_last_cuda_error) */
  ATTN_ERR_DEVICE = 7       /* a kernel recorded a runtime error (attn_device_status) */
} attn_status;

/* Version of this ABI; bumped when a signature or a semantic changes. */
int attn_abi_version(void);

/* Static, human-readable name of a status code (never NULL). */
const char* attn_status_string(int status);

/* The cudaError_t of the last failed CUDA call made by this library on the
 * calling thread (0 if none). */
int attn_last_cuda_error(void);

/*
 * attn_fwd -- fused attention forward (prefill).
 *
 *   q    [B, Hq,  N, d] bf16      queries
 *   k    [B, Hkv, N, d] bf16      keys
 *   v    [B, Hkv, N, d] bf16      values
 *   o    [B, Hq,  N, d] bf16      output (written), rounded to nearest-even
 *   lse  [B, Hq,  N]    float32   natural-log log-sum-exp of each row's scaled
 *                                 scores over its visible keys (written)
 *   d in {64, 128}; Hq % Hkv == 0, query head h reads KV head h / (Hq / Hkv)
 *   causal: 0 = every key visible, 1 = query i sees keys j <= i
 *   scale: multiplies Q K^T before the mask; must be finite and > 0
 *
 * Accumulation is fp32 (scores, softmax statistics, P V); P enters the second
 * product as bf16.  o/lse may not alias q/k/v.
 * Errors: ATTN_ERR_NULL, ATTN_ERR_SHAPE (sizes < 1, d not 64/128, Hq % Hkv,
 * causal not 0/1, bad scale, a dimension too large for 32-bit indexing),
 * ATTN_ERR_ALIGN, ATTN_ERR_LAUNCH.
 */
int attn_fwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o,
             float* lse, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
             void* stream);

/*
 * attn_fwd_window -- attn_fwd with a sliding window: query i sees the keys j
 * with i - window_left <= j (and j <= i when causal), i.e. the additive mask M
 * of the attention equation is also -inf left of the window.  The pattern is
 * named beside causal as a standard mask that keeps a fused path in use
 * ("Finding the Next One: Fusion Beyond Attention", anylearn.cc, on silent
 * fallbacks) and as the Longformer-style window of block-sparse attention
 * ("Kernel Fusion and Custom Kernels", ai.zenoagi.com, section 4 on
 * FlashInfer); no page fixes its size.  window_left = -1
 * means no left limit (attn_fwd is this call with -1); window_left = 0 with
 * causal = 1 lets each query see only itself.  KV tiles wholly outside every
 * row's window are skipped, so the work is O(N * window) instead of O(N^2).
 * Errors: those of attn_fwd, plus ATTN_ERR_SHAPE for window_left < -1.
 */
int attn_fwd_window(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o,
                    float* lse, int B, int Hq, int Hkv, int N, int d, int causal, int window_left,
                    float scale, void* stream);

/*
 * attn_fwd_block_sparse -- attn_fwd with a 2-D block-sparse mask (the
 * block-sparse masks of FlashInfer, e.g. Longformer's window-plus-global
 * pattern, "Kernel Fusion and Custom Kernels", ai.zenoagi.com, section 4):
 * key j is visible to query i only if block (i / 128, j / 128) is kept, on top
 * of the causal mask.  KV tiles of masked blocks are never loaded or computed.
 *   block_mask: uint64 words; query block qb of head (b, h) keeps KV block j
 *   iff bit j % 64 of word j / 64 is set in the row of ceil(ceil(N/128)/64)
 *   words at block_mask + b * mask_b_stride + h * mask_h_stride
 *   + qb * ceil(ceil(N/128)/64) (strides in words; 0 broadcasts; 8-byte
 *   aligned; bits past the last KV block are ignored).
 * A query row that sees no key at all gets O = 0 and LSE = -inf.  N <= 32768
 * (ATTN_ERR_UNSUPPORTED above).  Other arguments and errors as attn_fwd.
 */
int attn_fwd_block_sparse(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse,
                          int B, int Hq, int Hkv, int N, int d, int causal, float scale, const uint64_t* block_mask,
                          long long mask_b_stride, long long mask_h_stride, void* stream);

/*
 * attn_fwd_bias -- attn_fwd with a general additive mask M:
 * softmax(scale * Q K^T + M) V ("FlashAttention-Style Kernels", the attention
 * equation with M), M any finite values or -inf, added on top of the causal
 * mask when causal = 1.
 *   bias: bf16, natural-log units (the units of scale * q.k); M[i][j] of head
 *     (b, h) at bias + b * bias_b_stride + h * bias_h_stride
 *     + i * bias_row_stride + j (strides in elements, each >= 0 and a multiple
 *     of 8; 0 broadcasts, e.g. bias_row_stride = 0 for one key-padding row per
 *     head; bias 16-byte aligned).  Each row holds N values followed by
 *     padding up to a multiple of 8 elements (read, then ignored: any bits),
 *     so bias_row_stride, when not 0, is at least that padded length.
 *     Read-only; owned by the caller.
 * A query row whose scores are all -inf gets O = 0 and LSE = -inf.  +inf or
 * NaN in M gives undefined (but in-bounds) results.  Other arguments and
 * errors as attn_fwd; ATTN_ERR_SHAPE for negative or short strides,
 * ATTN_ERR_ALIGN for strides that are not multiples of 8.
 */
int attn_fwd_bias(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* o, float* lse, int B,
                  int Hq, int Hkv, int N, int d, int causal, float scale, const attn_bf16* bias,
                  long long bias_b_stride, long long bias_h_stride, long long bias_row_stride, void* stream);

/*
 * attn_fwd_fp8 -- attn_fwd with e4m3 inputs (OCP FP8 E4M3 codes, one byte
 * each, same [B, H, N, d] layouts): the attention of q * q_descale,
 * k * k_descale and v * v_descale, the FP8 tensor-core path of FlashAttention
 * v3 ("Kernel Fusion and Custom Kernels", ai.zenoagi.com, section 3
 * "FlashAttention: The Milestone of Fusion", under "v3 (2024,
 * H100-Exclusive)": Q K and P V computed in FP8 for twice the tensor-core
 * rate).  Q K^T and P V run on the FP8 tensor cores with fp32 accumulation;
 * P is rounded to e4m3 (scaled by 2^8) before P V, the row sums and LSE use
 * P unrounded.  o is bf16, lse fp32.
 * d must be 128 (ATTN_ERR_UNSUPPORTED for 64); the descales finite and > 0.
 * Error behaviour as attn_fwd.
 */
int attn_fwd_fp8(const uint8_t* q, const uint8_t* k, const uint8_t* v, attn_bf16* o, float* lse, int B, int Hq,
                 int Hkv, int N, int d, int causal, float scale, float q_descale, float k_descale, float v_descale,
                 void* stream);

/*
 * paged_attn_decode_split_tokens -- tokens per split of the split-KV decode
 * pass for this problem shape (a multiple of 16).  The split plan depends only
 * on these arguments, never on the sequence lengths, so the host never has to
 * read device memory.
 */
int paged_attn_decode_split_tokens(int num_seqs, int Hkv, int max_pages, int page_size);

/*
 * paged_attn_decode_workspace_bytes -- bytes of device scratch that
 * paged_attn_decode needs for these sizes: per (sequence, query head, split)
 * a partial output row of d fp32 values and one fp32 partial LSE.  Returns 0
 * for invalid sizes.
 */
size_t paged_attn_decode_workspace_bytes(int num_seqs, int Hq, int d, int max_pages, int page_size);

/*
 * paged_attn_decode -- one-query-per-sequence attention over a paged KV cache.
 *
 *   q            [num_seqs, Hq, d] bf16       the newest token of each sequence
 *   k_pool       [num_pages, page_size, Hkv, d] bf16
 *   v_pool       [num_pages, page_size, Hkv, d] bf16
 *   block_table  [num_seqs, max_pages] int32  logical page p of sequence s is
 *                physical page block_table[s][p]; entries past a sequence's
 *                ceil(seq_len / page_size) pages are never read (any value,
 *                e.g. -1); entries may repeat across sequences (shared pages)
 *   seq_lens     [num_seqs] int32, 1 <= seq_len <= max_pages * page_size; the
 *                query attends to all seq_len cached tokens (no mask)
 *   o            [num_seqs, Hq, d] bf16 (written)
 *   lse          [num_seqs, Hq] float32, natural log (written)
 *   page_size    a multiple of 16, at most 256
 *   d in {64, 128}; Hq % Hkv == 0 and Hq / Hkv <= 16
 *   workspace    device scratch of at least
 *                paged_attn_decode_workspace_bytes(num_seqs, Hq, d, max_pages,
 *                page_size) bytes, 16-byte aligned, owned by the caller; its
 *                contents on entry do not matter; concurrent calls need
 *                separate workspaces.
 *
 * Slots of a last page past seq_len may hold anything (NaN included) and do
 * not affect the result.  A table entry outside [0, num_pages) or a length
 * outside its range is reported through attn_device_status() (the affected
 * outputs are then unspecified; invalid lengths give O = 0, LSE = -inf).
 * Errors: ATTN_ERR_NULL, ATTN_ERR_SHAPE, ATTN_ERR_ALIGN, ATTN_ERR_WORKSPACE,
 * ATTN_ERR_UNSUPPORTED (page_size, group size), ATTN_ERR_LAUNCH.
 */
int paged_attn_decode(const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool,
                      const int32_t* block_table, const int32_t* seq_lens, int page_size,
                      attn_bf16* o, float* lse, int num_seqs, int Hq, int Hkv, int d,
                      int max_pages, int num_pages, float scale, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * ATTN_NOALLOC_SCRATCH_BYTES -- size of the device scratch array built into
 * the library for paged_attn_decode_noalloc (48 MiB).
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (48u * 1024u * 1024u)

/*
 * paged_attn_decode_noalloc -- paged_attn_decode for callers that cannot
 * allocate device memory.  The pages have no counterpart to this call: it is
 * a deployment convenience, not part of the method.
 *
 * Who needs it: a plug-in whose host program owns all device memory and does
 * not let plug-ins allocate; a latency-critical serving loop, where a
 * cudaMalloc may synchronise the device and stall other streams; a process
 * whose memory pool has already reserved everything.  Such callers pass the
 * same arguments as to paged_attn_decode minus the workspace, and the split
 * partials go to a fixed array of ATTN_NOALLOC_SCRATCH_BYTES compiled into
 * the library.  This call never calls cudaMalloc, cudaFree or any other
 * allocating routine.
 *
 * - Every GPU on which the library's device code is loaded keeps that array
 *   (48 MiB) until the process exits.  The CUDA runtime creates it when it
 *   loads the library's device code on a device; with lazy module loading
 *   (the default since CUDA 12.2) that happens inside the first call on that
 *   device, which then fails with ATTN_ERR_LAUNCH (attn_last_cuda_error()
 *   names the CUDA error, e.g. out of memory) if the device has no room left.
 *   Make one warm-up call at start-up, before memory is handed out.
 * - Limit: sizes whose paged_attn_decode_workspace_bytes() exceed
 *   ATTN_NOALLOC_SCRATCH_BYTES are refused with ATTN_ERR_WORKSPACE before any
 *   CUDA call, after the same argument checks as paged_attn_decode (a bad
 *   argument is reported as itself).  (The 64-sequence, 32-head,
 *   8192-token-table workload needs 33.8 MB.)
 * - The first call in each CUDA context of a device looks up the array's
 *   device address (cudaGetSymbolAddress) and caches it under the context's
 *   id; after a device reset the next call looks it up again.  Make the first
 *   call on a device (and the first after a reset) before any stream capture
 *   on that device.
 * - All calls on a device share the one array and it keeps whatever the last
 *   call left there (nothing in it needs to start at zero).  Calls whose
 *   kernels can overlap on the GPU (different streams, or different host
 *   threads without ordering) race on it and produce wrong results: order
 *   them on one stream, or use paged_attn_decode with separate workspaces.
 * Errors: those of paged_attn_decode, with ATTN_ERR_WORKSPACE meaning "larger
 * than the built-in scratch".
 */
int paged_attn_decode_noalloc(const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool,
                              const int32_t* block_table, const int32_t* seq_lens, int page_size,
                              attn_bf16* o, float* lse, int num_seqs, int Hq, int Hkv, int d,
                              int max_pages, int num_pages, float scale, void* stream);

/*
 * Decode as a CUDA graph -- the split pass and the merge of paged_attn_decode
 * captured once and replayed, which removes the per-call host work and launch
 * gaps that dominate small-batch decode ("Fast Attention Kernels and Operator
 * Fusion", section "Fusion and CUDA Graphs with torch.compile": a captured
 * graph is replayed with one submission; anylearn.cc: capture the decode step
 * once and replay it, removing per-launch cost).
 *
 * paged_attn_decode_graph_create takes exactly the arguments of
 * paged_attn_decode (minus the stream) and returns an opaque handle in *graph.
 * The graph keeps every pointer and size it was created with: between
 * launches the caller may change the CONTENTS of q, k_pool, v_pool,
 * block_table and seq_lens (same shapes; seq_lens within 1..max_pages *
 * page_size), and must keep all buffers, the workspace included, alive until
 * the handle is destroyed.  Creation synchronises nothing but does allocate
 * host and device resources for the graph; it fails with the status
 * paged_attn_decode would return for bad arguments.
 * paged_attn_decode_graph_launch enqueues one decode step on `stream`.
 * paged_attn_decode_graph_destroy frees the handle (NULL is allowed); the
 * caller must make sure no launch of it is still running.
 */
typedef struct attn_decode_graph attn_decode_graph;

int paged_attn_decode_graph_create(const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool,
                                   const int32_t* block_table, const int32_t* seq_lens, int page_size,
                                   attn_bf16* o, float* lse, int num_seqs, int Hq, int Hkv, int d,
                                   int max_pages, int num_pages, float scale, void* workspace,
                                   size_t workspace_bytes, attn_decode_graph** graph);
int paged_attn_decode_graph_launch(attn_decode_graph* graph, void* stream);
int paged_attn_decode_graph_destroy(attn_decode_graph* graph);

/*
 * Appending to a paged cache, and chunked (paged) prefill.
 *
 * A step hands each sequence s a chunk of q_len(s) new tokens, packed by
 * sequence: rows cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1 of q [total_q, Hq, d]
 * and of k_new / v_new [total_q, Hkv, d] (cu_seqlens_q [num_seqs+1] int32,
 * non-decreasing, cu_seqlens_q[0] = 0, cu_seqlens_q[num_seqs] <= total_q).
 * seq_lens [num_seqs] int32 is each sequence's length AFTER the step, so the
 * chunk is logical tokens ctx .. seq_len-1 with ctx = seq_len - q_len, and
 * the pools, block table, page_size, max_pages and num_pages are as for
 * paged_attn_decode (pages for all seq_len tokens already assigned in the
 * table: "blocks can be allocated on demand", "Fast Attention Kernels and
 * Operator Fusion", section "Paged Attention Kernels").  page_size must be
 * 16, 32, 64, 128 or 256.  A sequence whose lengths are out of range, or a
 * table entry outside the pool, is skipped and reported through
 * attn_device_status (bit 12); nothing is written outside the outputs and the
 * pool slots of valid chunks.
 *
 * paged_kv_append -- writes new token i of sequence s (its K and V rows, all
 * Hkv heads) to physical page block_table[s][(ctx + i) / page_size], slot
 * (ctx + i) % page_size: the cache update the same page lists among the
 * fusions of a layer (section "Operator Fusion").  Exact copies.  Every other
 * pool slot is left as it was.
 */
int paged_kv_append(const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_pool, attn_bf16* v_pool,
                    const int32_t* cu_seqlens_q, const int32_t* seq_lens, const int32_t* block_table,
                    int num_seqs, int total_q, int Hkv, int d, int page_size, int max_pages, int num_pages,
                    void* stream);

/*
 * paged_prefill -- attention of every sequence's new queries over its whole
 * paged cache (the chunk included, so call it after paged_kv_append, or use
 * paged_prefill_append).  New query i of sequence s is token ctx + i: with
 * causal = 1 it sees keys 0 .. ctx + i, with causal = 0 all seq_len keys.
 *   o    [total_q, Hq, d] bf16 (written: rows of valid chunks)
 *   lse  [total_q, Hq] float32, natural log (written likewise)
 * The same fused kernel as attn_fwd (scores stay on chip), with K/V read
 * through the block table one page at a time; slots past a sequence's end
 * are never used, whatever they hold.  d in {64, 128}, Hq % Hkv == 0,
 * num_seqs <= 1024 and (total_q + 255 * num_seqs) / 256 <= 2048 (at most 2048
 * query blocks of 256 rows; ATTN_ERR_UNSUPPORTED beyond).  No workspace.
 */
int paged_prefill(const attn_bf16* q, const attn_bf16* k_pool, const attn_bf16* v_pool,
                  const int32_t* cu_seqlens_q, const int32_t* seq_lens, const int32_t* block_table, attn_bf16* o,
                  float* lse, int num_seqs, int total_q, int Hq, int Hkv, int d, int page_size, int max_pages,
                  int num_pages, int causal, float scale, void* stream);

/*
 * paged_prefill_append -- paged_kv_append followed by paged_prefill on the
 * same stream, one call: the chunk's keys and values go into their pages and
 * the attention then reads everything, the chunk included, through the table.
 * All arguments are checked before either kernel is enqueued.
 */
int paged_prefill_append(const attn_bf16* q, const attn_bf16* k_new, const attn_bf16* v_new, attn_bf16* k_pool,
                         attn_bf16* v_pool, const int32_t* cu_seqlens_q, const int32_t* seq_lens,
                         const int32_t* block_table, attn_bf16* o, float* lse, int num_seqs, int total_q, int Hq,
                         int Hkv, int d, int page_size, int max_pages, int num_pages, int causal, float scale,
                         void* stream);

/*
 * attn_device_status -- synchronises `stream`, then reads and clears the
 * device error word of the current device.  Returns ATTN_OK if no kernel
 * recorded an error since the last call, ATTN_ERR_DEVICE otherwise (the raw
 * bit mask is stored in *bits when bits != NULL), ATTN_ERR_LAUNCH if the
 * synchronisation itself failed.
 */
int attn_device_status(void* stream, unsigned int* bits);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* ATTN_B200_H */
