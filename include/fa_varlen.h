/*
 * fa_varlen.h -- C ABI of the B200 (sm_100a) variable-length attention
 * library, libfa_varlen.so.
 *
 * What it computes. Exact scaled-dot-product attention over a batch of
 * sequences packed back to back without padding, addressed by cumulative
 * offsets, forward and backward, with an optional causal mask:
 *
 *   for each sequence b and head h, with Q_b = q[cu_seqlens_q[b] :
 *   cu_seqlens_q[b+1], h, :] and K_b, V_b taken likewise from cu_seqlens_k,
 *     S = softmax_scale * Q_b K_b^T, masked entries excluded,
 *     lse_i = log sum_j exp(S_ij)          (natural log, scaled scores),
 *     out   = exp(S - lse) V_b.
 *
 * Sources: the page "Mecanismo cu_seqlens en FlashAttention" (friki.work),
 * sections "Estructuras de datos clave" (the offsets arrays hold batch+1
 * cumulative offsets; [0,128,300] means lengths 128 and 172), "Lógica de
 * cálculo de longitud" (length = cu[b+1] - cu[b]) and "Optimización de
 * acceso a memoria" (a sequence starts at packed row cu[b]); the page
 * "FlashAttention na inferência" (slavadubrov.com), section "Separar o
 * armazenamento do cálculo" (exact attention: score every visible pair,
 * normalise, multiply by V; computed here blockwise with an online softmax,
 * never materialising S in memory); the page "FlashAttention-2 GPU work
 * partitioning" (iplexlaw.co.kr), section "Bloques pequeños, normalización
 * global" (global normalisation; results equal up to floating-point order);
 * the page "Flash-Atención y Flash-Atención-2" (zepes.com), FlashAttention v1
 * and backward sections (the backward recomputes the probabilities; column
 * blocks are independent workers and the query gradient is aggregated with
 * atomic additions).
 *
 * Causal mask. Key j of a sequence is visible from its query i iff
 *   j <= i + (lk - lq)        (bottom-right alignment; for lq == lk this is
 *                              the usual j <= i).
 * A query row with no visible key gets out = 0 and lse = -inf.
 *
 * Layouts (all row-major, contiguous, device memory):
 *   q, out, dout, dq : bf16 [total_q, num_heads, head_dim]
 *   k, v, dk, dv     : bf16 [total_k, num_heads, head_dim]
 *   softmax_lse      : fp32 [num_heads, total_q]
 *   cu_seqlens_q/k   : int32 [batch + 1], device memory, cu[0] = 0,
 *                      non-decreasing, cu[batch] = total_q / total_k.
 * Element (row, h, c) of a packed tensor is at (row*num_heads + h)*head_dim + c.
 *
 * Supported head dimensions (anything else returns FA_ERR_UNSUPPORTED;
 * there is no fallback path):
 *   - 64 and 128 on every entry point;
 *   - 256 on the forwards (fa_varlen_fwd, _gqa, _kvcache, _paged, _noalloc)
 *     and the backwards (fa_varlen_bwd, _gqa, _deterministic); the split-KV
 *     forward (fa_varlen_fwd_splitkv) refuses it.
 * The page "Flash-Atención y Flash-Atención-2" (FlashAttention-2 section)
 * gives head dimensions "up to 256"; this library reads that as the three
 * powers of two 64, 128 and 256 that tile into whole 64-column (128-byte)
 * swizzled chunks. q, k, v, out, dout, dq, dk, dv must be 16-byte aligned.
 * softmax_scale must be finite and > 0.
 *
 * Ownership and synchrony. The caller owns every buffer, including the
 * workspace (size from the *_workspace_size functions, any 256-byte-aligned
 * device allocation). Calls only enqueue work on `stream` and return; they
 * never synchronise. The library keeps no state between calls. Calls are
 * thread-safe; two calls that run concurrently must not share a workspace.
 *
 * Errors. The return value reports argument validation and launch errors.
 * Errors found on the device (malformed cu_seqlens, a wait that timed out)
 * are written to a status word in the workspace; every kernel of the call
 * then exits early and the outputs are undefined. fa_get_device_status reads
 * that word.
 */
#ifndef FA_VARLEN_H
#define FA_VARLEN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Identical to cudaStream_t (the CUDA runtime's stream handle). */
struct CUstream_st;
typedef struct CUstream_st* fa_cuda_stream_t;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative size, bad scale, misaligned pointer */
  FA_ERR_UNSUPPORTED = 2,      /* head_dim not supported by the entry point, or sizes beyond the limits below */
  FA_ERR_WORKSPACE = 3,        /* workspace null, misaligned or smaller than required */
  FA_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed */
  FA_ERR_BAD_SEQLENS = 5,      /* device: cu_seqlens not monotone, cu[0] != 0, cu[batch] != total,
                                  or a length above max_seqlen */
  FA_ERR_DEVICE_TIMEOUT = 6    /* device: a pipeline wait gave up after its time limit */
} fa_status_t;

/* Limits (FA_ERR_UNSUPPORTED beyond them): num_heads * head_dim < 2^31;
 * total_q and total_k below 2^31 - 256; (total_q / 128 + batch + 1) *
 * num_heads and (total_k / 128 + batch + 1) * num_heads below 2^31. */

/* Workspace bytes needed by fa_varlen_fwd for these sizes. */
size_t fa_varlen_fwd_workspace_size(int batch, int total_q, int num_heads, int head_dim);

/* Workspace bytes needed by fa_varlen_bwd for these sizes (includes an fp32
 * dQ accumulator of about total_q * num_heads * head_dim * 4 bytes). */
size_t fa_varlen_bwd_workspace_size(int batch, int total_q, int total_k, int num_heads, int head_dim);

/* Forward. Writes out and softmax_lse for every row of every sequence.
 * max_seqlen_q / max_seqlen_k bound the sequence lengths (checked on the
 * device). Rows of out/softmax_lse outside [0, total_q) are never written. */
fa_status_t fa_varlen_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                          const int32_t* cu_seqlens_k, int batch, int total_q, int total_k, int max_seqlen_q,
                          int max_seqlen_k, int num_heads, int head_dim, float softmax_scale, int causal,
                          void* out, float* softmax_lse, void* workspace, size_t workspace_bytes,
                          fa_cuda_stream_t stream);

/* Backward of L = sum(out * dout) given the forward's out and softmax_lse.
 * Recomputes the probabilities from softmax_lse; writes dq, dk, dv.
 * The query gradient is accumulated with fp32 atomic reductions, so dq may
 * differ in the last bits between runs (fa_varlen_bwd_deterministic does
 * not). head_dim 64, 128 or 256; at 256 the work runs as two passes over
 * the same work list (dv first, then dk and dq), which the caller does not
 * see: the arguments, workspace size and results are the same. */
fa_status_t fa_varlen_bwd(const void* dout, const void* q, const void* k, const void* v, const void* out,
                          const float* softmax_lse, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                          int batch, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int num_heads,
                          int head_dim, float softmax_scale, int causal, void* dq, void* dk, void* dv,
                          void* workspace, size_t workspace_bytes, fa_cuda_stream_t stream);

/* Grouped-query and multi-query attention (page "Flash-Atención y
 * Flash-Atención-2", FlashAttention-2 section: several query heads attend to
 * one key/value head, which shrinks the key/value cache). Same as
 * fa_varlen_fwd / fa_varlen_bwd, except that k, v, dk and dv have
 * num_heads_k heads:
 *   k, v, dk, dv : bf16 [total_k, num_heads_k, head_dim]
 * num_heads must be a multiple of num_heads_k (else FA_ERR_INVALID_ARGUMENT);
 * query head h reads key/value head h / (num_heads / num_heads_k), i.e.
 * consecutive query heads share one (the pages do not say which heads share;
 * this is the mapping of repeating each key/value head over its group).
 * dk and dv of a shared head are the sums over its query heads, accumulated
 * on chip (no atomic additions). num_heads_k == num_heads is exactly
 * fa_varlen_fwd / fa_varlen_bwd. The workspace sizes are those of
 * fa_varlen_fwd_workspace_size / fa_varlen_bwd_workspace_size with the query
 * head count. */
fa_status_t fa_varlen_fwd_gqa(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                              const int32_t* cu_seqlens_k, int batch, int total_q, int total_k, int max_seqlen_q,
                              int max_seqlen_k, int num_heads, int num_heads_k, int head_dim, float softmax_scale,
                              int causal, void* out, float* softmax_lse, void* workspace, size_t workspace_bytes,
                              fa_cuda_stream_t stream);
fa_status_t fa_varlen_bwd_gqa(const void* dout, const void* q, const void* k, const void* v, const void* out,
                              const float* softmax_lse, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                              int batch, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                              int num_heads, int num_heads_k, int head_dim, float softmax_scale, int causal,
                              void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                              fa_cuda_stream_t stream);

/* Deterministic backward (same arguments and results as fa_varlen_bwd_gqa).
 * The page "Flash-Atención y Flash-Atención-2" (backward paragraph) has the
 * column workers aggregate the query gradient with atomic additions, whose
 * order, and so whose rounding, changes from run to run. Here every 128-row
 * query tile receives its dQ contributions in key-tile order: key tile j
 * waits (on a per-tile counter in the workspace) until key tiles 0 .. j-1
 * have added theirs. dq, dk and dv are then bitwise identical from run to
 * run for the same inputs, sizes and GPU model. The work list is taken in
 * (sequence, key tile) order rather than longest first, so the call is
 * somewhat slower than fa_varlen_bwd_gqa. A wait that does not end within
 * its time limit is reported as FA_ERR_DEVICE_TIMEOUT in the workspace
 * status. Workspace: fa_varlen_bwd_workspace_size. */
fa_status_t fa_varlen_bwd_deterministic(const void* dout, const void* q, const void* k, const void* v,
                                        const void* out, const float* softmax_lse, const int32_t* cu_seqlens_q,
                                        const int32_t* cu_seqlens_k, int batch, int total_q, int total_k,
                                        int max_seqlen_q, int max_seqlen_k, int num_heads, int num_heads_k,
                                        int head_dim, float softmax_scale, int causal, void* dq, void* dk, void* dv,
                                        void* workspace, size_t workspace_bytes, fa_cuda_stream_t stream);

/* Forward over a key/value cache: the keys of each sequence are given by a
 * per-sequence length instead of cumulative offsets, optionally after some
 * left padding (page "Mecanismo cu_seqlens en FlashAttention", "Lógica de
 * cálculo de longitud": the key array may be non-cumulative, and the cache
 * length of a sequence is its key count minus its left padding).
 *   k_cache, v_cache : bf16 [batch, cache_rows, num_heads_k, head_dim]; slot b
 *                      holds sequence b's keys at rows leftpad_k[b] ..
 *                      seqlens_k[b]-1, so it has lk = seqlens_k[b] - leftpad_k[b]
 *                      keys (rows outside that range are never read).
 *   seqlens_k        : int32 [batch], device memory.
 *   leftpad_k        : int32 [batch], device memory, or NULL (no padding).
 * Queries, out and softmax_lse are packed with cu_seqlens_q exactly as in
 * fa_varlen_fwd; the causal rule uses lq and lk as defined here (key j of
 * the valid range is visible from query i iff j <= i + lk - lq). Grouped
 * heads as in fa_varlen_fwd_gqa. The workspace size is
 * fa_varlen_fwd_workspace_size(batch, total_q, num_heads, head_dim).
 * Errors: FA_ERR_INVALID_ARGUMENT for a null seqlens_k; on the device,
 * FA_ERR_BAD_SEQLENS unless 0 <= leftpad_k[b] <= seqlens_k[b] <= cache_rows
 * for every b (besides the checks of cu_seqlens_q); batch * cache_rows must
 * stay below 2^31 - 256 rows (FA_ERR_UNSUPPORTED). There is no backward for
 * this layout. */
fa_status_t fa_varlen_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* cu_seqlens_q, const int32_t* seqlens_k, const int32_t* leftpad_k,
                                  int batch, int total_q, int cache_rows, int max_seqlen_q, int num_heads,
                                  int num_heads_k, int head_dim, float softmax_scale, int causal, void* out,
                                  float* softmax_lse, void* workspace, size_t workspace_bytes,
                                  fa_cuda_stream_t stream);

/* Forward over a paged key/value cache (the pages' "caché KV paginada", on
 * the cu_seqlens page, section "Integración con máscaras causales y caché
 * paginada"): keys and values sit in a pool of fixed-size pages and each
 * sequence lists its pages in a block table.
 *   k_pages, v_pages : bf16 [num_pages, page_size, num_heads_k, head_dim]
 *   seqlens_k        : int32 [batch], device: sequence b has seqlens_k[b]
 *                      keys, key position p in page block_table[b][p /
 *                      page_size] at row p % page_size.
 *   block_table      : int32 [batch, max_pages_per_seq], device, row-major;
 *                      entries past a sequence's last page are not read.
 * page_size must be a multiple of 128 (FA_ERR_UNSUPPORTED otherwise: a key
 * tile of 128 rows is then always inside one page). max_seqlen_k bounds
 * seqlens_k. Queries, outputs, causal rule and grouped heads as in
 * fa_varlen_fwd_gqa; workspace as fa_varlen_fwd_workspace_size(batch,
 * total_q, num_heads, head_dim). On the device, FA_ERR_BAD_SEQLENS unless
 * 0 <= seqlens_k[b] <= min(max_seqlen_k, max_pages_per_seq * page_size)
 * and every page a sequence uses is in [0, num_pages). There is no backward
 * for this layout. */
fa_status_t fa_varlen_fwd_paged(const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* cu_seqlens_q, const int32_t* seqlens_k, const int32_t* block_table,
                                int batch, int total_q, int num_pages, int page_size, int max_pages_per_seq,
                                int max_seqlen_q, int max_seqlen_k, int num_heads, int num_heads_k, int head_dim,
                                float softmax_scale, int causal, void* out, float* softmax_lse, void* workspace,
                                size_t workspace_bytes, fa_cuda_stream_t stream);

/* Where the keys and values of each sequence live, for
 * fa_varlen_fwd_splitkv (exactly one of the three layouts):
 *  - packed: cu_seqlens_k [batch+1] cumulative offsets (as fa_varlen_fwd);
 *  - key/value cache slots: seqlens_k, leftpad_k (or NULL), cache_rows (as
 *    fa_varlen_fwd_kvcache; k and v are [batch * cache_rows, Hk, d]);
 *  - paged cache: seqlens_k, block_table, page_size (a multiple of 128),
 *    max_pages_per_seq (as fa_varlen_fwd_paged; k and v are
 *    [num_pages * page_size, Hk, d]).
 * total_rows is the number of rows of k and v. All pointers are device
 * memory; unused fields are NULL / 0. */
typedef struct {
  const int32_t* cu_seqlens_k;
  const int32_t* seqlens_k;
  const int32_t* leftpad_k;
  const int32_t* block_table;
  int cache_rows;
  int page_size;
  int max_pages_per_seq;
  int total_rows;
} fa_kv_layout_t;

/* Split-KV forward for decoding and other short-query calls (the page
 * "FlashAttention-2 GPU work partitioning", section "Cómo documentar una
 * diferencia técnica", separates prefill from token-by-token decoding, whose
 * bottleneck differs). Same results as fa_varlen_fwd_gqa (and the cache
 * forwards) for any num_splits; the work decomposition differs:
 *  - the g = num_heads / num_heads_k query heads that share a key/value head
 *    (g <= 128) and 128 / g consecutive query tokens of a sequence form one
 *    128-row tile, so each key/value tile is read once per group;
 *  - each tile's key tiles are divided into num_splits ranges processed in
 *    parallel; each writes a normalised partial output and its logsumexp
 *    into the workspace (fp32) and a combine kernel merges them
 *    (num_splits = 1 writes out directly).
 * head_dim 64 or 128 (FA_ERR_UNSUPPORTED otherwise). The workspace must
 * hold fa_varlen_fwd_splitkv_workspace_size(...) bytes (0 = invalid sizes).
 * Layout-specific checks are those of the matching entry point. When
 * max_seqlen_q <= floor(128 / g) (every sequence fits one tile: decoding)
 * the call builds no work list: it resets the workspace's status word and
 * work counters with one cudaMemsetAsync and the decode kernel checks each
 * sequence as it takes its work; a sequence that fails a check is skipped
 * and FA_ERR_BAD_SEQLENS is recorded (the outputs are then undefined, as
 * for every device-side error). */
size_t fa_varlen_fwd_splitkv_workspace_size(int batch, int total_q, int num_heads, int num_heads_k, int head_dim,
                                            int num_splits);
fa_status_t fa_varlen_fwd_splitkv(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                                  const fa_kv_layout_t* kv, int batch, int total_q, int max_seqlen_q,
                                  int max_seqlen_k, int num_heads, int num_heads_k, int head_dim, float softmax_scale,
                                  int causal, int num_splits, void* out, float* softmax_lse, void* workspace,
                                  size_t workspace_bytes, fa_cuda_stream_t stream);

/* A split count for fa_varlen_fwd_splitkv (advisory; results do not depend
 * on it). The work units of the split-KV forward are (sequence, key/value
 * head, query tile, key range), taken by one persistent CTA per SM. This
 * returns the smallest num_splits for which the units fill the SMs in
 * nearly whole waves (at least 95% of the CTA-unit slots busy, the units
 * being of equal size), keeping at least two 128-key tiles per range; if no
 * count reaches that, the one with the best fill. If that count leaves
 * fewer than 8 key tiles per range, where a unit's fixed costs dominate, it
 * returns instead the smallest count whose units occupy at least 85% of the
 * SMs at once, when there is a smaller one. A query tile holds
 * tq = floor(128 / group) tokens of one sequence (group = num_heads /
 * num_heads_k), so the unit count per range is taken as
 * batch * num_heads_k * ceil(max_seqlen_q / tq).
 * sm_count <= 0 uses the current device's SM count. Returns 1 for invalid
 * arguments or when no device can be queried. Host only; no device work. */
int fa_varlen_splitkv_num_splits(int batch, int max_seqlen_q, int num_heads, int num_heads_k, int max_seqlen_k,
                                 int sm_count);

/* Forward for callers that cannot allocate device memory. The pages have no
 * counterpart of this entry point; it exists for the library's users.
 *
 * Same arguments and results as fa_varlen_fwd, without the workspace. Some
 * callers cannot call cudaMalloc: code running inside another framework's
 * plugin or operator interface that receives only input and output pointers
 * (allocating outside that framework's pool breaks its accounting), or
 * latency-critical paths where a device allocation, which may synchronise
 * the device, is not allowed. This entry point allocates nothing: its scratch
 * is a library-owned device buffer of FA_NOALLOC_SCRATCH_BYTES (256 KiB) that
 * every GPU loading the library holds until the process exits.
 *
 * - Returns FA_ERR_WORKSPACE, before any CUDA call, when the sizes need more
 *   scratch than that: fa_varlen_fwd_workspace_size(batch, total_q,
 *   num_heads, head_dim) must not exceed FA_NOALLOC_SCRATCH_BYTES. That size
 *   is about 256 + 4 * batch + 8 * (total_q / item_rows + batch) bytes,
 *   item_rows being the query rows of one work item (256 for head_dim 64 and
 *   128, 128 for head_dim 256), so total_q / item_rows + 1.5 * batch must
 *   stay below about 32600.
 * - The first call on each device (and the first after a device reset, which
 *   creates a new context) looks up the buffer's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 * - All calls on a device share the one buffer, which keeps the last call's
 *   contents: calls that can overlap on the GPU (different streams, or
 *   different host threads) race and must be serialised by the caller.
 * - Errors found on the device (malformed cu_seqlens) cannot be read back:
 *   the outputs are then undefined. */
#define FA_NOALLOC_SCRATCH_BYTES (256u * 1024u)
fa_status_t fa_varlen_fwd_noalloc(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                                  const int32_t* cu_seqlens_k, int batch, int total_q, int total_k,
                                  int max_seqlen_q, int max_seqlen_k, int num_heads, int head_dim,
                                  float softmax_scale, int causal, void* out, float* softmax_lse,
                                  fa_cuda_stream_t stream);

/* Synchronises `stream`, then returns the device-side status of the last
 * call that used `workspace` (FA_OK, FA_ERR_BAD_SEQLENS or
 * FA_ERR_DEVICE_TIMEOUT), or FA_ERR_CUDA if the synchronisation failed. */
fa_status_t fa_get_device_status(const void* workspace, fa_cuda_stream_t stream);

/* Measurement hook for benchmarks; normal callers never need it. With
 * `events` non-null, every later fa_varlen_fwd / fa_varlen_bwd call made from
 * the calling host thread records, on its stream, events[2i] just before and
 * events[2i+1] just after the i-th kernel it launches (i counts from 0 in each
 * call; forward: 0 work-list preparation, 1 attention; backward: 0 work-list
 * preparation, 1 preprocess, 2 attention gradients, 3 dQ conversion), for
 * i < n_pairs. `events` holds cudaEvent_t handles created by the caller and
 * must stay valid while the hook is on. Pass NULL to turn it off. */
void fa_set_kernel_events(void* const* events, int n_pairs);

/* Test hook for the device-side failure detection; normal callers never need
 * it. It applies to every later call made from the calling host thread.
 * wait_limit_ns: the time after which every pipeline wait in the kernels
 * gives up, records FA_ERR_DEVICE_TIMEOUT in the workspace status and makes
 * the CTA stop (0 restores the default, 2 s). withhold_first_value_load != 0:
 * the forward (fa_varlen_fwd, _gqa, _kvcache, _paged at head_dim 64 or 128)
 * never issues the first value-tile load of its first work item and never
 * posts that load's byte count, so the wait for it runs out; no load or MMA
 * is left in flight, the call's outputs are undefined and the workspace
 * status reads FA_ERR_DEVICE_TIMEOUT. The next call on the same workspace
 * starts from a clean status. fa_set_test_hooks(0, 0) turns both off. */
void fa_set_test_hooks(uint64_t wait_limit_ns, int withhold_first_value_load);

/* Static, human-readable name of a status code. */
const char* fa_status_string(fa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* FA_VARLEN_H */
