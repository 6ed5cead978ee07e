/*
 * fa.h -- C ABI of libfa.so: exact, IO-aware multi-head attention on B200 (sm_100a).
 *
 * The operation is exact attention, O = softmax(scale * Q K^T) V, per batch
 * element and head ("FlashAttention saves IO, not N^2 work", section 1:
 * S = QK^T / sqrt(d), P = softmax(S), O = PV).  It is computed tile by tile
 * with an online softmax so that the N x N score and probability matrices never
 * reach device memory (same page, sections 2-3; Flash Attention wiki note,
 * "Online Softmax" and "Tiling").  The backward pass recomputes S and P from the
 * saved per-row log-sum-exp ("AI Bible 13", section 03, second axe: keep only O
 * and the row statistics).  Decode splits each row's KV history into chunks and
 * merges the chunks' (m, l, u) states (first page, sections 3 and 7; section 6
 * for the decode shapes).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers, 16-byte aligned, contiguous, in the
 *    layouts stated per call.  bf16 means IEEE bfloat16 (2 bytes).
 *  - The caller owns every buffer, including `workspace`.  The library never
 *    allocates device memory, never keeps a pointer after returning, and never
 *    synchronises the device (except fa_check).
 *  - Work is enqueued asynchronously on `stream` (0 = legacy default stream).
 *    Launch failures are returned as FA_ERR_CUDA; the CUDA error is consumed.
 *  - Supported head dimensions: d in {64, 128}.  Only bf16 inputs/outputs.
 *  - softmax_scale <= 0 selects 1/sqrt(d).
 *  - causal != 0 applies a bottom-right aligned mask: query row i (of Nq) sees
 *    key j (of Nk) iff j <= i + (Nk - Nq).  A query row that sees no key gets
 *    O = 0 and LSE = -inf (and zero gradients).  For decode (one query row) the
 *    mask admits every key and is a no-op.
 *  - LSE is the natural-log log-sum-exp of the scaled scores of a row:
 *    lse_i = m_i + ln(l_i), with m_i the row max and l_i = sum_j exp(s_ij - m_i).
 *  - A workspace must be zero-filled (cudaMemset) before its first use.  After
 *    that the library keeps it consistent by itself and it may be reused for
 *    any shape: fa_check clears the status word, and the decode merge tickets
 *    sit at a fixed place and reset themselves.  After fa_check has reported
 *    FA_ERR_TIMEOUT, zero the workspace again before reusing it.  Two calls
 *    that may run at the same time on the GPU must not share a workspace.
 *  - Every wait inside a kernel is bounded (default about 2 s; environment
 *    variable FA_WAIT_TIMEOUT_MS overrides it).  A wait that runs out makes the
 *    kernel record FA_ERR_TIMEOUT in the workspace's status word and return
 *    without further work; fa_check reports it.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, Nq != 1 for decode, ... */
  FA_ERR_UNSUPPORTED = 2, /* head dimension or configuration this build does not implement */
  FA_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned */
  FA_ERR_WORKSPACE = 4,   /* workspace null or smaller than the *_workspace_size query */
  FA_ERR_CUDA = 5,        /* a CUDA runtime/driver call or kernel launch failed */
  FA_ERR_TIMEOUT = 6      /* a kernel's bounded wait ran out (reported by fa_check) */
} fa_status;

/*
 * Forward pass.
 *   q   : [B, Nq, H, d] bf16 (token-major, d innermost)
 *   k, v: [B, Nk, H, d] bf16
 *   o   : [B, Nq, H, d] bf16 (written)
 *   lse : [B, H, Nq]    fp32 (written) -- saved for the backward pass
 *   workspace: at least fa_fwd_workspace_size(...) bytes of device memory,
 *              16-byte aligned; holds the kernel status word.
 * Sizes: B, H, Nq, Nk >= 1; d in {64, 128}.  q/k/v must not alias o/lse.
 * Returns FA_OK when the work was enqueued.
 */
FA_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int Nq, int Nk, int d, int causal, float softmax_scale, void* workspace,
                 size_t workspace_bytes, cudaStream_t stream);

/*
 * Forward pass over a batch of sequences of different lengths, packed without
 * padding (the variable-length prefill of the paging / padding discussion,
 * "FlashAttention saves IO, not N^2 work", section 6).  Same computation as
 * fa_fwd, sequence by sequence; the causal mask is bottom-right aligned within
 * each sequence.
 *   q, o        : [total_q, H, d] bf16; sequence b owns rows
 *                 cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 *   k, v        : [total_k, H, d] bf16, rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1
 *   cu_seqlens_q, cu_seqlens_k : device int32 [B+1], non-decreasing, starting at 0
 *   lse         : [H, total_q] fp32 (written)
 *   max_seqlen_q, max_seqlen_k : upper bounds of the sequence lengths (lengths
 *                 above them are cut to them)
 *   workspace   : at least fa_fwd_workspace_size(...) bytes (the status word)
 * A sequence whose offsets do not fit the buffers is skipped and recorded in
 * the status word (fa_check then returns FA_ERR_INVALID_ARG); no store leaves
 * the rows of its own sequence.  Rows of a sequence with no keys get O = 0 and
 * LSE = -inf.
 */
FA_API fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                               const int32_t* cu_seqlens_k, void* o, float* lse, int B, int H,
                               int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                               int causal, float softmax_scale, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/*
 * Backward pass (recompute form).
 *   q, o, do_ : [B, Nq, H, d] bf16 ; k, v : [B, Nk, H, d] bf16
 *   lse       : [B, H, Nq] fp32 as written by fa_fwd with the same arguments
 *   dq        : [B, Nq, H, d] bf16 (written)
 *   dk, dv    : [B, Nk, H, d] bf16 (written)
 *   workspace : at least fa_bwd_workspace_size(...) bytes; holds an fp32 dQ
 *               accumulator [B, Nq, H, d], the row terms D_i = dO_i . O_i
 *               [B, H, Nq] fp32, and the status word.  The call clears the dQ
 *               accumulator itself.
 * Gradients are of the scalar sum(O * dO) with respect to q, k and v.  The dq
 * accumulation uses fp32 atomics, so dq is reproducible only up to summation
 * order.
 */
FA_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* do_,
                 const float* lse, void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int d,
                 int causal, float softmax_scale, void* workspace, size_t workspace_bytes,
                 cudaStream_t stream);

/*
 * Backward pass of fa_fwd_varlen: the gradients of sum(O * dO) over a packed
 * batch, sequence by sequence (the recompute form of fa_bwd; "AI Bible 13",
 * section 03).
 *   q, o, do_, dq : [total_q, H, d] bf16 (dq written), rows of sequence b are
 *                   cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 *   k, v, dk, dv  : [total_k, H, d] bf16 (dk, dv written), rows
 *                   cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1
 *   lse           : [H, total_q] fp32 as written by fa_fwd_varlen with the same
 *                   arguments
 *   cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k : as fa_fwd_varlen
 *   workspace     : at least fa_bwd_varlen_workspace_size(H, total_q, d) bytes
 *                   (fp32 dQ accumulator [total_q, H, d], D [H, total_q], status)
 * dK and dV of a sequence with no queries are zero, as is dQ of a sequence with
 * no keys.  dq rows past the last sequence are zero; dk / dv rows past the last
 * sequence are not written.  Offsets that do not fit the buffers are handled as
 * in fa_fwd_varlen (skipped, FA_ERR_INVALID_ARG from fa_check).
 */
FA_API fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* do_,
                               const float* lse, void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q,
                               const int32_t* cu_seqlens_k, int B, int H, int total_q, int total_k,
                               int max_seqlen_q, int max_seqlen_k, int d, int causal, float softmax_scale,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Forward and backward passes with a key-padding mask and dropout (the padding
 * mask and dropout the pages list among the semantics a fused attention kernel has
 * to match, "FlashAttention saves IO, not N^2 work", section 8; both inside the one
 * kernel, with dropout's mask generated again in the backward pass rather than
 * stored, "AI Bible 13", section 03).  Arguments, layouts and results are those of
 * fa_fwd and fa_bwd, plus
 *   key_mask  : device uint32 [B, (Nk + 31) / 32], 4-byte aligned, or NULL for no
 *               mask; bit j % 32 of word j / 32 is set when key j of batch element
 *               b takes part.  A masked key is excluded like a causally masked one
 *               (both apply when both are set; the causal alignment still counts
 *               all Nk keys).  A row left with no key gets O = 0 and LSE = -inf; a
 *               masked key gets dK = dV = 0.  Bits past key Nk - 1 are ignored.
 *   dropout_p : probability of dropping each (query, key) probability, 0 <= p < 1
 *               (rounded to t / 65536 with t = round(65536 p); FA_ERR_INVALID_ARG
 *               outside that range).  The output is O = (P o Z) V with Z = keep /
 *               (1 - t / 65536), P the softmax of the unmasked keys; LSE stays that
 *               of the undropped softmax.
 *   seed      : 64-bit seed of the dropout draws.  Element (b, h, i, j) uses
 *               Philox4x32-10 (Salmon et al., SC'11) keyed by the seed (low word
 *               first) with counter (j / 2, i / 4, h, b): word i % 4, low 16 bits
 *               for even j, high 16 bits for odd j; kept when those bits >= t.
 * The backward pass takes the same key_mask, dropout_p and seed as its forward,
 * and that forward's O and LSE.  NULL key_mask with dropout_p = 0 makes the calls
 * fa_fwd and fa_bwd.
 */
FA_API fa_status fa_fwd_masked(const void* q, const void* k, const void* v, void* o, float* lse,
                               const uint32_t* key_mask, float dropout_p, unsigned long long seed, int B, int H,
                               int Nq, int Nk, int d, int causal, float softmax_scale, void* workspace,
                               size_t workspace_bytes, cudaStream_t stream);
FA_API fa_status fa_bwd_masked(const void* q, const void* k, const void* v, const void* o, const void* do_,
                               const float* lse, void* dq, void* dk, void* dv, const uint32_t* key_mask,
                               float dropout_p, unsigned long long seed, int B, int H, int Nq, int Nk, int d,
                               int causal, float softmax_scale, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/*
 * Block-sparse forward and backward passes (the block-sparse variant "AI Bible 13",
 * section 05, credits with the 64K-token results): attention restricted to the
 * (query tile, key tile) blocks a mask keeps.  Arguments, layouts and results are
 * those of fa_fwd and fa_bwd, plus
 *   block_mask : device uint8 [H, ceil(Nq / 128), ceil(Nk / 128)] (shared by the
 *                batch), not NULL; block (i, j) of head h covers query rows
 *                128 i .. 128 i + 127 and keys 128 j .. 128 j + 127, and a 0 removes
 *                all of its keys from all of its queries (on top of the causal
 *                mask).  Blocks that are 0 are not computed, and a key tile that no
 *                query tile of a work item keeps is not loaded.  A row
 *                left with no key gets O = 0 and LSE = -inf; keys that no kept block
 *                reaches get dK = dV = 0.
 * The backward pass takes the same block_mask as its forward.
 */
FA_API fa_status fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                                    const uint8_t* block_mask, int B, int H, int Nq, int Nk, int d, int causal,
                                    float softmax_scale, void* workspace, size_t workspace_bytes,
                                    cudaStream_t stream);
FA_API fa_status fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o, const void* do_,
                                    const float* lse, void* dq, void* dk, void* dv, const uint8_t* block_mask, int B,
                                    int H, int Nq, int Nk, int d, int causal, float softmax_scale, void* workspace,
                                    size_t workspace_bytes, cudaStream_t stream);

/*
 * Causal attention over one shard of the keys, for causal sequence parallelism:
 * the shard k, v [B, Nk, H, d] holds keys key_offset .. key_offset + Nk - 1 of a
 * sequence of Nk_total keys, and query i (of Nq, all queries) sees shard key j iff
 * key_offset + j <= i + (Nk_total - Nq) (the bottom-right alignment of the whole
 * sequence).  Layouts and results as fa_fwd / fa_bwd with causal = 1; merge the
 * shards' forward results with fa_merge_partials, and run the backward of each
 * shard with the merged O and LSE.  A query row that sees no key of the shard gets
 * O = 0 and LSE = -inf from fa_fwd_shard, and shard keys no query sees get
 * dK = dV = 0.  FA_ERR_INVALID_ARG unless 0 <= key_offset and
 * key_offset + Nk <= Nk_total.
 */
FA_API fa_status fa_fwd_shard(const void* q, const void* k, const void* v, void* o, float* lse, int key_offset,
                              int Nk_total, int B, int H, int Nq, int Nk, int d, float softmax_scale, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream);
FA_API fa_status fa_bwd_shard(const void* q, const void* k, const void* v, const void* o, const void* do_,
                              const float* lse, void* dq, void* dk, void* dv, int key_offset, int Nk_total, int B,
                              int H, int Nq, int Nk, int d, float softmax_scale, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream);

/*
 * Merge of partial attention results over key shards, for sequence parallelism
 * (the multi-GPU extension the second page wishes for, "AI Bible 13", section 06):
 * when the keys and values are split into S shards and fa_fwd runs over each shard
 * with all queries (not causal; causal shards go through fa_fwd_shard), the shard
 * results combine by the block-merge rule
 * ("FlashAttention saves IO, not N^2 work", sections 3 and 7):
 *     O = sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M),  M = max_s lse_s,
 *     lse = M + ln sum_s exp(lse_s - M).
 *   o_parts   : [S, B, Nq, H, d] bf16, shard s's fa_fwd output at o_parts + s * B Nq H d
 *   lse_parts : [S, B, H, Nq] fp32, shard s's lse
 *   o, lse    : [B, Nq, H, d] bf16 and [B, H, Nq] fp32 (written)
 * A shard with lse = -inf for a row contributes nothing to it; a row with no key in
 * any shard gets O = 0 and LSE = -inf.  No workspace; 16-byte aligned pointers.
 * The backward of sequence-parallel attention needs no merge: fa_bwd over each
 * shard with the merged O and lse gives that shard's dK and dV exactly and a
 * partial dQ, and the partial dQ sum over shards is dQ.
 */
FA_API fa_status fa_merge_partials(const void* o_parts, const float* lse_parts, int S, int B, int H, int Nq, int d,
                                   void* o, float* lse, cudaStream_t stream);

/*
 * Split-KV decode over a ragged, packed KV cache.
 *   q           : [B, H, d] bf16 (one query row per sequence: Nq must be 1)
 *   k, v        : [total_kv, H, d] bf16; sequence b owns rows
 *                 cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1
 *   cu_seqlens_k: device int32 [B+1], non-decreasing, cu_seqlens_k[0] = 0,
 *                 cu_seqlens_k[B] <= total_kv.  This is a precondition: the
 *                 call has no total_kv to check the last bound against, and
 *                 offsets that break it make the kernel read outside k and v.
 *                 FA_CHECKS=1 checks the order on the device first.  Callers
 *                 whose offsets come from untrusted data use
 *                 fa_decode_splitkv_checked, which checks them against total_kv.
 *   max_seqlen_k: an upper bound of every sequence length (plays the role of Nk)
 *   num_splits  : chunks per sequence; 0 picks a value from the shape
 *   o           : [B, H, d] bf16 (written);  lse : [B, H] fp32 (written)
 *   workspace   : at least fa_decode_workspace_size(B, H, max_seqlen_k, d, num_splits)
 *                 bytes; holds the per-chunk (m, l, u) partial states, the merge
 *                 tickets and the status word.
 * A sequence of length 0 gets O = 0 and LSE = -inf.
 */
FA_API fa_status fa_decode_splitkv(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_k,
                            int B, int H, int Nq, int max_seqlen_k, int d, int causal,
                            float softmax_scale, int num_splits, void* o, float* lse, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_decode_splitkv with the number of rows of k and v, so that the offsets can
 * be checked on the device instead of being a precondition.  Same computation,
 * layouts and workspace as fa_decode_splitkv.
 *   total_kv : rows of k and v ([total_kv, H, d]); >= 0, else FA_ERR_INVALID_ARG
 * A sequence b whose rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1 do not lie in
 * [0, total_kv) (a negative start, an end before its start, or an end past
 * total_kv) is skipped before any of its rows is read: its o and lse are left
 * as they were, and the kernel records the fault in the workspace status word
 * (fa_check then returns FA_ERR_INVALID_ARG).  The other sequences are computed
 * as usual.
 */
FA_API fa_status fa_decode_splitkv_checked(const void* q, const void* k, const void* v,
                                           const int32_t* cu_seqlens_k, int B, int H, int Nq, int total_kv,
                                           int max_seqlen_k, int d, int causal, float softmax_scale,
                                           int num_splits, void* o, float* lse, void* workspace,
                                           size_t workspace_bytes, cudaStream_t stream);

/*
 * Split-KV decode over a paged KV cache (the paging the pages name as the
 * batched-decode layout question, "FlashAttention saves IO, not N^2 work",
 * section 6).  Same computation as fa_decode_splitkv; only the cache layout
 * differs.
 *   q                : [B, H, d] bf16, one query row per sequence
 *   k_pages, v_pages : [num_pages, page_size, H, d] bf16 (any page_size >= 1)
 *   block_table      : device int32 [B, max_pages_per_seq]; key t of sequence b is
 *                      row t % page_size of page block_table[b][t / page_size].
 *                      Entries past a sequence's last page are not read.
 *   seqlens_k        : device int32 [B], keys per sequence; values are clamped to
 *                      [0, max_seqlen_k]
 *   max_seqlen_k     : an upper bound of every sequence length; must not exceed
 *                      max_pages_per_seq * page_size (FA_ERR_INVALID_ARG)
 *   num_splits, o, lse, workspace: as for fa_decode_splitkv (same workspace size)
 * A page index outside [0, num_pages) is never dereferenced: the kernel records
 * it in the workspace status word (fa_check then returns FA_ERR_INVALID_ARG) and
 * reads page 0 in its place, so that output is meaningless but nothing outside
 * the cache is touched.  A sequence of length 0 gets O = 0 and LSE = -inf.
 */
FA_API fa_status fa_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                 const int32_t* block_table, const int32_t* seqlens_k, int B, int H,
                                 int num_pages, int page_size, int max_pages_per_seq, int max_seqlen_k,
                                 int d, float softmax_scale, int num_splits, void* o, float* lse,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_decode_splitkv without a workspace, for callers that cannot allocate
 * device memory -- for example an operator inside a host framework that owns
 * every device allocation and offers it no allocator, or a serving loop that
 * must never call cudaMalloc (which may synchronise the device).  The pages
 * have no counterpart of this call; it exists for such callers only.
 *
 * Arguments, layouts and results are those of fa_decode_splitkv.  The chunk
 * states live instead in a scratch array of 16 MiB compiled into the library,
 * which every GPU that loads the library holds until the process exits.
 *  - The call allocates nothing.  Its first call on a device looks up the
 *    array's device address (cudaGetSymbolAddress, with that device current);
 *    make that first call before any stream capture.  With lazy module loading
 *    that first lookup is also when the CUDA runtime loads the library's device
 *    code and places the array, which may allocate and synchronise: make the
 *    first call outside any latency-critical loop.  The address is kept for the
 *    life of the process, so the device must not be reset (cudaDeviceReset)
 *    after the first call.
 *  - FA_CHECKS=1 and FA_WAIT_TIMEOUT_MS act as for fa_decode_splitkv.
 *  - Returns FA_ERR_WORKSPACE when the shape needs more than the 16 MiB of
 *    scratch (B * H * splits * (d + 2) * 4 bytes plus small overheads); pass a
 *    smaller num_splits then.
 *  - All calls share the one array, and each call clears the parts that must
 *    start at zero.  Calls whose kernels may overlap on the GPU (concurrent
 *    streams, several host threads) therefore race: serialise them.
 *  - Bounded waits still end a stuck kernel, but there is no workspace for
 *    fa_check, so this call does not report FA_ERR_TIMEOUT.
 */
FA_API fa_status fa_decode_splitkv_noalloc(const void* q, const void* k, const void* v,
                                           const int32_t* cu_seqlens_k, int B, int H, int Nq,
                                           int max_seqlen_k, int d, int causal, float softmax_scale,
                                           int num_splits, void* o, float* lse, cudaStream_t stream);

/* Workspace sizes in bytes for the calls above (0 when the arguments are invalid). */
FA_API size_t fa_fwd_workspace_size(int B, int H, int Nq, int Nk, int d);
FA_API size_t fa_bwd_workspace_size(int B, int H, int Nq, int Nk, int d);
FA_API size_t fa_bwd_varlen_workspace_size(int H, int total_q, int d);
FA_API size_t fa_decode_workspace_size(int B, int H, int max_seqlen_k, int d, int num_splits);

/*
 * Number of KV chunks per sequence that fa_decode_splitkv uses for these
 * arguments (num_splits = 0 resolves to the automatic choice).
 */
FA_API int fa_decode_num_splits(int B, int H, int max_seqlen_k, int d, int num_splits);

/*
 * Synchronises `stream` and reads the status word that the kernels of the
 * previous call(s) with this workspace recorded, then clears it.  Returns FA_OK,
 * FA_ERR_TIMEOUT (a bounded wait ran out), FA_ERR_INVALID_ARG (an argument the
 * kernels found bad: variable-length or checked-decode offsets outside the
 * buffers, a paged-decode page index outside the cache, or, with FA_CHECKS=1,
 * decode cu_seqlens out of order) or FA_ERR_CUDA.
 */
FA_API fa_status fa_check(void* workspace, cudaStream_t stream);

/*
 * Self-test of the failure path (no counterpart in the pages).  Launches one
 * thread that waits, with the library's bounded wait, on a barrier nothing
 * arrives on; after `timeout_us` microseconds (1 .. 1000000) the wait gives up
 * and records FA_ERR_TIMEOUT in the workspace status word, exactly as a stuck
 * kernel would.  A following fa_check on the same workspace returns
 * FA_ERR_TIMEOUT and clears the word; the context stays usable.
 */
FA_API fa_status fa_selftest_wait_timeout(void* workspace, size_t workspace_bytes, unsigned timeout_us,
                                          cudaStream_t stream);

/* Human-readable name of a status code (static string). */
FA_API const char* fa_status_string(fa_status status);

/* Library version as "major.minor.patch" (static string). */
FA_API const char* fa_version(void);

/*
 * Launch profiling (off by default; the pages ask for evidence of which kernel
 * actually ran -- "FlashAttention saves IO, not N^2 work", section 8).
 * Between fa_profile_start and fa_profile_stop every kernel the library
 * launches is bracketed by a pair of CUDA events on its stream.  fa_profile_stop
 * waits for those events and totals them per kernel; fa_profile_get then
 * returns, for kernel index `id` in [0, fa_profile_count()), its name, the number
 * of launches and their summed device time in milliseconds.  Returns FA_OK, or
 * FA_ERR_INVALID_ARG for a bad index, FA_ERR_CUDA when an event call failed.
 * The events are driver objects created on first use and kept for reuse; no
 * device memory is allocated.  Profiling is process-wide and not meant for
 * concurrent use from several threads.
 */
FA_API fa_status fa_profile_start(void);
FA_API fa_status fa_profile_stop(void);
FA_API int fa_profile_count(void);
FA_API fa_status fa_profile_get(int id, const char** name, int* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
