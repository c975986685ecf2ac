/*
 * mla.h -- C ABI of the B200 (sm_100a) multi-head latent attention library.
 *
 * The operation is DeepSeek-V3 multi-head latent attention in its "absorb"
 * form, as set out in "Naive vs Absorb Attention Implementations in
 * DeepSeek-V3", section "Absorb Path Execution":
 *
 *   W       = wkv_b viewed as [H, Dn + Dv, C]      (rows 0..Dn-1: key part,
 *                                                   rows Dn..Dn+Dv-1: value part)
 *   q_abs   = q_nope . W[:, :Dn]                    mla_absorb_q
 *   scores  = (q_abs . kv^T + q_pe . pe^T) * scale  mla_attn_decode /
 *   P       = softmax over keys (causal, aligned    mla_attn_prefill_chunk
 *             to the end of the cache)
 *   o_lat   = P . kv
 *   out     = o_lat . W[:, Dn:]^T                   mla_out_proj
 *
 * The cache layout is the page's absorb cache design ("Absorb Implementation
 * Cache Design"): kv_cache holds the compressed latent (C = kv_lora_rank
 * values per token) and pe_cache the rotary key (R = qk_rope_head_dim values
 * per token); neither has a head axis.  Here sequences are packed one after
 * another along the token axis and located by cu_seqlens (an exclusive
 * prefix sum of per-sequence lengths, batch + 1 entries, device memory).
 *
 * Conventions common to every call:
 *  - Every pointer argument except `dims` and the `*_out` results is a
 *    DEVICE pointer owned by the caller; the library never allocates, frees
 *    or synchronises on these calls.  All calls are asynchronous on `stream`
 *    and keep no state between calls, so they may be issued from several
 *    host threads on different streams.
 *  - Element types follow dims->dtype: MLA_DTYPE_BF16 (bfloat16 storage,
 *    fp32 accumulation) or MLA_DTYPE_F32 (fp32 throughout).  cu_seqlens are
 *    int32.
 *  - Device buffers must be 16-byte aligned.
 *  - The host checks sizes, alignment and the workspace before launching and
 *    returns a status without launching on failure.  Sequence lengths live on
 *    the device and are not read by the host: a negative length is treated
 *    as 0, and a query row that sees no key gets zeros.
 *  - Device-side waits are bounded.  A wait that runs out sets a device
 *    error word instead of trapping; mla_device_status reports it.
 *  - mla_attn_paged reads the same caches through a block table instead
 *    (pages of page_size tokens); its description gives the addressing.
 *  - Early start.  The tensor-core kernels (bf16 DeepSeek-V3 shapes) are
 *    launched with programmatic dependent launch: a kernel may start while
 *    the kernel before it on the stream is finishing, and reads what that
 *    kernel may write (q, q_abs, o_lat, ...) and writes its outputs only
 *    after waiting for it.  Before that wait it reads only inputs that do
 *    not change from one step of a model to the next or that the step has
 *    already written: mla_absorb_q and mla_out_proj read wkv_b, and the
 *    attention calls (decode, decode_out, decode_fused, decode_partials,
 *    decode_static_scratch, prefill_chunk, paged) read kv_cache, pe_cache,
 *    cu_seqlens_q, cu_seqlens_k, seqlens_k and block_table.  These must not
 *    be written by the kernel launched just before the call on the same
 *    stream, unless that kernel makes its writes visible device-wide before
 *    it exits (mla_append_latent does: append -> attention is safe).  A
 *    copy (cudaMemcpyAsync) or an event between the two is always safe.
 */
#ifndef MLA_B200_H_
#define MLA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t; 0 is the legacy default stream. */
#ifndef __DRIVER_TYPES_H__
typedef struct CUstream_st* cudaStream_t;
#endif

#define MLA_API_VERSION 1

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

typedef enum mla_status {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,     /* null pointer, bad size, misaligned pointer, bad stride */
  MLA_ERR_UNSUPPORTED = 2,     /* dims not compiled in (see each call) */
  MLA_ERR_WORKSPACE = 3,       /* workspace missing or smaller than mla_workspace_size */
  MLA_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed */
  MLA_ERR_DEVICE_TIMEOUT = 5   /* a bounded device wait ran out (see mla_device_status) */
} mla_status_t;

typedef enum mla_dtype { MLA_DTYPE_BF16 = 0, MLA_DTYPE_F32 = 1 } mla_dtype_t;

/* Head geometry.  H = num_heads, C = kv_lora_rank, Dn = qk_nope_head_dim,
 * R = qk_rope_head_dim, Dv = v_head_dim.  softmax_scale multiplies the scores
 * (DeepSeek-V3 without YaRN: 1/sqrt(Dn + R)); it must be finite and >= 0
 * (calls with other values return MLA_ERR_UNSUPPORTED).
 *
 * bf16 runs on the tcgen05 tensor-core kernels when C = 512, R = 64,
 * Dn = Dv = 128 and H is a multiple of 128 (the DeepSeek-V3 shapes); other
 * bf16 shapes and every fp32 shape run on CUDA-core kernels, which need
 * C <= 1024, R <= 128, Dn <= 256, Dv <= 256 and H <= 1024. */
typedef struct mla_dims {
  int32_t num_heads;
  int32_t kv_lora_rank;
  int32_t qk_nope_head_dim;
  int32_t qk_rope_head_dim;
  int32_t v_head_dim;
  int32_t dtype;        /* mla_dtype_t */
  float softmax_scale;
} mla_dims_t;

/* Absorbed query: q_abs[n,h,c] = sum_{d<Dn} q[n,h,d] * wkv_b[h*(Dn+Dv)+d, c].
 * ("Absorb Path Execution", the einsum that folds q_nope through the key
 * rows of wkv_b.)
 *   q        [n_rows, H, Dn+R], row n starts at q + n*q_row_stride elements,
 *            head h of a row at + h*(Dn+R); only dims 0..Dn-1 are read.
 *   wkv_b    [H*(Dn+Dv), C] row-major.
 *   q_abs    [n_rows, H, C] contiguous, written.
 *   n_rows   >= 0 (0 is a no-op).  q_row_stride >= H*(Dn+R).  The tensor-core
 *            kernels take at most 65535 * 256 rows per call (MLA_ERR_INVALID_ARG above). */
MLA_API mla_status_t mla_absorb_q(const mla_dims_t* dims, const void* q, int64_t q_row_stride,
                          const void* wkv_b, void* q_abs, int64_t n_rows, cudaStream_t stream);

/* Bytes of workspace mla_attn_decode / mla_attn_prefill_chunk need for these
 * sizes.  num_splits = 0 means the automatic choice the attention call makes
 * for the same arguments.  n_q_rows = total query rows (batch for decode). */
MLA_API size_t mla_workspace_size(const mla_dims_t* dims, int32_t batch, int64_t n_q_rows,
                          int64_t max_seqlen_k, int32_t num_splits);

/* Number of key-range splits mla_attn_decode uses for these arguments
 * (num_splits = 0: the automatic choice).  With more than one split the
 * call launches a merge kernel after the attention kernel. */
MLA_API int32_t mla_decode_num_splits(const mla_dims_t* dims, int32_t batch, int64_t max_seqlen_k,
                                      int32_t num_splits);

/* Decode attention: one query per sequence over its whole cache (no mask).
 * ("Absorb Path Execution", the score einsums and the latent value einsum;
 * the softmax between them is the reading documented with the oracle.)
 *   q_abs        [batch, H, C] (from mla_absorb_q).
 *   q            [batch, H, Dn+R] with row stride q_row_stride; the rotary
 *                part q_pe is read from dims Dn..Dn+R-1.
 *   kv_cache     [kv_rows, C], pe_cache [kv_rows, R]; sequence b owns rows
 *                cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1.
 *   kv_rows      host count of rows in both cache buffers (>= cu_seqlens_k[batch]);
 *                nothing past it is read (sequence ranges are clamped to it).
 *   cu_seqlens_k device int32 [batch+1], non-decreasing.
 *   max_seqlen_k host upper bound of every sequence length (keys past it
 *                are not read); it sizes the split-t partition.
 *   o_lat        [batch, H, C] written: softmax-weighted sum of latent rows.
 *   workspace    device scratch of at least mla_workspace_size(dims, batch,
 *                batch, max_seqlen_k, num_splits) bytes (may be NULL when
 *                that is 0).  Contents on entry are ignored.
 *   num_splits   0 = automatic; otherwise the key range of each sequence is
 *                cut into that many parts that are merged afterwards (1..256).
 */
MLA_API mla_status_t mla_attn_decode(const mla_dims_t* dims, const void* q_abs, const void* q,
                             int64_t q_row_stride, const void* kv_cache, const void* pe_cache,
                             int64_t kv_rows, const int32_t* cu_seqlens_k, int32_t batch, int64_t max_seqlen_k,
                             void* o_lat, void* workspace, size_t workspace_bytes,
                             int32_t num_splits, cudaStream_t stream);

/* Bytes of workspace mla_attn_decode_out needs (num_splits as there; 0 = automatic). */
MLA_API size_t mla_decode_out_workspace_size(const mla_dims_t* dims, int32_t batch, int64_t max_seqlen_k,
                                             int32_t num_splits);

/* Decode attention followed by the output projection in one call:
 *   out[b,h,d] = sum_c o_lat[b,h,c] * wkv_b[h*(Dn+Dv)+Dn+d, c]
 * with o_lat as mla_attn_decode computes it ("Absorb Path Execution": the
 * score and latent value einsums, then the last einsum).  Arguments as in
 * mla_attn_decode, except:
 *   wkv_b      [H*(Dn+Dv), C], the same matrix mla_absorb_q and mla_out_proj take.
 *   out        [batch, H, Dv] contiguous, written.
 *   workspace  at least mla_decode_out_workspace_size(dims, batch, max_seqlen_k,
 *              num_splits) bytes, 16-byte aligned; o_lat lives there and is not
 *              returned.  Contents on entry are ignored.
 * The result equals mla_attn_decode followed by mla_out_proj, bit for bit.
 * On the tensor-core path with more than one split, the split merge runs
 * inside the projection kernel: o_lat never goes to memory and one kernel
 * launch is saved.  The wkv_b rule of mla_out_proj applies. */
MLA_API mla_status_t mla_attn_decode_out(const mla_dims_t* dims, const void* q_abs, const void* q,
                                         int64_t q_row_stride, const void* kv_cache, const void* pe_cache,
                                         int64_t kv_rows, const int32_t* cu_seqlens_k, int32_t batch,
                                         int64_t max_seqlen_k, const void* wkv_b, void* out, void* workspace,
                                         size_t workspace_bytes, int32_t num_splits, cudaStream_t stream);

/* Bytes of workspace mla_attn_decode_partials needs (num_splits as for
 * mla_attn_decode; 0 = automatic).  0 for dims the call does not support. */
MLA_API size_t mla_partials_workspace_size(const mla_dims_t* dims, int32_t batch, int64_t max_seqlen_k,
                                           int32_t num_splits);

/* Decode attention without the split merge: the per-split partial results are
 * left in the workspace for the caller to combine (a caller that spreads one
 * sequence's key range over several GPUs merges partials from all of them).
 * ("Absorb Path Execution", the score and latent value einsums over one key
 * range each; the merge rule below is the log-sum-exp combination of
 * softmaxes over disjoint key ranges.)  Arguments as in mla_attn_decode,
 * without o_lat.  With S = mla_decode_num_splits(dims, batch, max_seqlen_k,
 * num_splits), the workspace then holds, for split s of sequence b and head h:
 *   O[s, b, h, 0..C-1]  bf16 at byte 0: sum over the split's keys j of
 *                       2^(x_j - m) kv[j], where x_j = score_j * scale * log2(e);
 *   (m, l)[s, b, h]     two fp32 at byte offset align256(S * batch * H * C * 2):
 *                       m = the split's reference (>= max_j x_j - 8 when the split
 *                       has keys), l = sum_j 2^(x_j - m);
 * and o_lat[b, h] = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s with
 * M = max_s m_s.  A split without keys has m = -inf, l = 0 and leaves its O
 * rows unwritten.  Only the tensor-core kernels have this form (bf16
 * DeepSeek-V3 shapes); other dims return MLA_ERR_UNSUPPORTED.
 *   workspace  at least mla_partials_workspace_size(dims, batch, max_seqlen_k,
 *              num_splits) bytes, 16-byte aligned. */
MLA_API mla_status_t mla_attn_decode_partials(const mla_dims_t* dims, const void* q_abs, const void* q,
                                              int64_t q_row_stride, const void* kv_cache, const void* pe_cache,
                                              int64_t kv_rows, const int32_t* cu_seqlens_k, int32_t batch,
                                              int64_t max_seqlen_k, void* workspace, size_t workspace_bytes,
                                              int32_t num_splits, cudaStream_t stream);

/* Merge of split partials into o_lat: o_lat[n, h] = sum_s 2^(m_s - M) O_s /
 * sum_s 2^(m_s - M) l_s, M = max_s m_s (the log-sum-exp combination of
 * softmaxes over disjoint key ranges; "Absorb Path Execution", the latent
 * value einsum summed over the ranges).  The partials are in the form
 * mla_attn_decode_partials leaves them, and may come from several such calls
 * over disjoint key ranges of the same query rows, stacked along the split
 * axis (e.g. the parts of one long sequence held by several GPUs, gathered):
 *   part_o   [num_splits, n_q_rows, H, C] bf16 (O relative to each split's m)
 *   part_ml  [num_splits, n_q_rows, H, 2] fp32 (m, l); a split with m = -inf
 *            (no key) contributes nothing and its O rows are not read.
 *   o_lat    [n_q_rows, H, C] bf16, written.  A row whose splits all have
 *            l = 0 gets zeros.
 * 1 <= num_splits <= 256.  Tensor-core dims (bf16 DeepSeek-V3 shapes) only;
 * other dims return MLA_ERR_UNSUPPORTED. */
MLA_API mla_status_t mla_merge_partials(const mla_dims_t* dims, const void* part_o, const void* part_ml,
                                        int32_t num_splits, int64_t n_q_rows, void* o_lat, cudaStream_t stream);

/* The same merge fused into the output projection (as mla_attn_decode_out
 * does): out[n, h, :] = o_lat[n, h, :] . W_v[h]^T with o_lat never written.
 *   wkv_b  [H*(Dn+Dv), C] row-major; out [n_q_rows, H, Dv] bf16, written.
 * The kernel reads wkv_b before waiting for the previous kernel on the stream
 * (see "Early start" above). */
MLA_API mla_status_t mla_merge_partials_out(const mla_dims_t* dims, const void* part_o, const void* part_ml,
                                            int32_t num_splits, int64_t n_q_rows, const void* wkv_b, void* out,
                                            cudaStream_t stream);

/* Bytes of workspace mla_attn_decode_fused needs (num_splits as for
 * mla_attn_decode; 0 = automatic). */
MLA_API size_t mla_decode_fused_workspace_size(const mla_dims_t* dims, int32_t batch, int64_t max_seqlen_k,
                                               int32_t num_splits);

/* mla_attn_decode_out in one kernel where it fits: the attention, the split
 * merge and the output projection ("Absorb Path Execution": the score and
 * latent value einsums, then the last einsum) run as one grid, each CTA
 * loading its head's value rows of wkv_b while the other units finish, then
 * merging and projecting once every unit's partials are in memory (a
 * grid-wide counter with a bounded wait).  Arguments and result as for
 * mla_attn_decode_out (bit-identical output), except the workspace:
 *   workspace  at least mla_decode_fused_workspace_size(dims, batch,
 *              max_seqlen_k, num_splits) bytes, 16-byte aligned.  Its first
 *              256 bytes are control words that MUST be zero when the
 *              workspace is first used (zero-fill it once after allocating);
 *              every call leaves them zero.  The rest is scratch whose
 *              contents on entry are ignored.  Calls that share a workspace
 *              must not overlap on the GPU.
 * The one-kernel form needs more than one split and every CTA resident at
 * once (2 x batch x splits x H/128 CTAs at most the number of SMs); other
 * calls, and the CUDA-core family, run mla_attn_decode_out's kernels on the
 * same workspace.  The wkv_b rule of mla_out_proj applies. */
MLA_API mla_status_t mla_attn_decode_fused(const mla_dims_t* dims, const void* q_abs, const void* q,
                                           int64_t q_row_stride, const void* kv_cache, const void* pe_cache,
                                           int64_t kv_rows, const int32_t* cu_seqlens_k, int32_t batch,
                                           int64_t max_seqlen_k, const void* wkv_b, void* out, void* workspace,
                                           size_t workspace_bytes, int32_t num_splits, cudaStream_t stream);

/* Size of the device scratch array behind mla_attn_decode_static_scratch. */
#define MLA_STATIC_SCRATCH_BYTES (32u << 20)

/* mla_attn_decode without a caller-provided workspace.  The method as
 * described has no counterpart to this call; it exists for callers that cannot allocate
 * device memory: code that only receives input and output buffers from a
 * host framework with no allocator to call, and code on a path where
 * cudaMalloc is not allowed or would synchronise the device (inside a
 * stream capture in global mode, a latency-bound decode loop).
 *
 * Arguments are those of mla_attn_decode minus the workspace.  The split-t
 * partials go to one library-owned device array of MLA_STATIC_SCRATCH_BYTES
 * per GPU, held from the library's first use on that GPU until the process
 * exits.  The call allocates and frees nothing.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - If the split plan needs more than MLA_STATIC_SCRATCH_BYTES (as
 *     mla_workspace_size would report), the call returns MLA_ERR_WORKSPACE
 *     and launches nothing; pass a smaller num_splits or use mla_attn_decode.
 *   - Every call on a device shares the array and leaves its partials there;
 *     nothing in it needs to start at zero.  Calls that overlap on the GPU
 *     (other streams, other host threads) race on it: serialise them. */
MLA_API mla_status_t mla_attn_decode_static_scratch(const mla_dims_t* dims, const void* q_abs, const void* q,
                                                    int64_t q_row_stride, const void* kv_cache,
                                                    const void* pe_cache, int64_t kv_rows,
                                                    const int32_t* cu_seqlens_k, int32_t batch,
                                                    int64_t max_seqlen_k, void* o_lat, int32_t num_splits,
                                                    cudaStream_t stream);

/* Chunked-prefill attention: sequence b has s_b = cu_seqlens_q[b+1]-cu_seqlens_q[b]
 * new queries whose keys are already the last s_b rows of its cache of
 * t_b rows; query i (0-based) sees keys j <= t_b - s_b + i.
 *   q_abs, q     [total_q, H, C] and [total_q, H, Dn+R] (row stride q_row_stride).
 *   cu_seqlens_q device int32 [batch+1]; cu_seqlens_k, kv_cache, pe_cache,
 *                kv_rows as for decode.
 *   max_seqlen_q, max_seqlen_k  host upper bounds of s_b and t_b.
 *   o_lat        [total_q, H, C] written.
 *   workspace    at least mla_workspace_size(dims, batch, total_q, max_seqlen_k, 0)
 *                bytes, where total_q = cu_seqlens_q[batch] <= n_q_rows given there.
 *   n_q_rows     host value of cu_seqlens_q[batch] (rows of q_abs / o_lat). */
MLA_API mla_status_t mla_attn_prefill_chunk(const mla_dims_t* dims, const void* q_abs, const void* q,
                                    int64_t q_row_stride, const int32_t* cu_seqlens_q,
                                    const int32_t* cu_seqlens_k, int32_t batch, int64_t n_q_rows,
                                    int64_t max_seqlen_q, int64_t max_seqlen_k,
                                    const void* kv_cache, const void* pe_cache, int64_t kv_rows, void* o_lat,
                                    void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Chunked-prefill attention on the naive path: per-head attention over keys
 * and values expanded from the latent cache (by mla_expand_kv), with the
 * rotary key shared by all heads.  ("Naive vs Absorb Attention
 * Implementations in DeepSeek-V3", section "Naive Path Execution"; "Latent
 * KV expansion with split" produces K_nope and V.)  For query i of the s_b new
 * queries of sequence b (t_b keys; query i sees keys j <= t_b - s_b + i):
 *   out[n,h,:] = sum_j softmax_j((q_nope[n,h] . K_nope[h,j] + q_pe[n,h] . pe[j]) * scale) V[h,j,:]
 * which equals mla_attn_prefill_chunk followed by mla_out_proj in exact
 * arithmetic (the pages' "mathematically identical" paths).
 *   q          [n_q_rows, H, Dn+R] with row stride q_row_stride (nope first).
 *   k_nope     [H, kv_rows, Dn] and v [H, kv_rows, Dv]: mla_expand_kv with
 *              batch = 1, seq_len = kv_rows over the packed compressed cache
 *              writes exactly this layout.
 *   pe_cache   [kv_rows, R]; sequence b owns key rows cu_seqlens_k[b] ..
 *              cu_seqlens_k[b+1]-1 of all three.
 *   cu_seqlens_q, cu_seqlens_k, n_q_rows, max_seqlen_q as for mla_attn_prefill_chunk.
 *   out        [n_q_rows, H, Dv] written (the attention output; no latent
 *              projection follows).
 * Needs no workspace.  Only the tensor-core kernels have this path (bf16
 * DeepSeek-V3 shapes); other dims return MLA_ERR_UNSUPPORTED. */
MLA_API mla_status_t mla_attn_prefill_expanded(const mla_dims_t* dims, const void* q, int64_t q_row_stride,
                                               const void* k_nope, const void* v, const void* pe_cache,
                                               int64_t kv_rows, const int32_t* cu_seqlens_q,
                                               const int32_t* cu_seqlens_k, int32_t batch, int64_t n_q_rows,
                                               int64_t max_seqlen_q, void* out, cudaStream_t stream);

/* Attention over a PAGED latent cache, decode or chunked prefill.
 * ("What is DeepSeek Sparse Attention (DSA)?", section "How DSA works
 * (conceptual)": the serving runtime keeps the KV cache in pages for
 * continuous batching.)  Same arithmetic as mla_attn_decode (cu_seqlens_q
 * NULL) and mla_attn_prefill_chunk (cu_seqlens_q given); only the addressing
 * of the cache differs:
 *   key j of sequence b sits in row  block_table[b * max_pages_per_seq + j / page_size]
 *                                    * page_size + j % page_size
 *   of kv_cache [num_pages * page_size, C] and pe_cache [num_pages * page_size, R].
 *   seqlens_k        device int32 [batch]: keys of each sequence (the current
 *                    token included); a length is capped at
 *                    max_pages_per_seq * page_size.
 *   block_table      device int32 [batch, max_pages_per_seq] row-major.  Only
 *                    the entries of pages that hold keys are read.  Such an
 *                    entry outside [0, num_pages) reads as a page of zeros and
 *                    sets bit 1<<7 of the device error word (mla_device_status
 *                    then returns MLA_ERR_DEVICE_TIMEOUT with that code).
 *   page_size        > 0; the tensor-core kernels need a multiple of 64
 *                    (others return MLA_ERR_UNSUPPORTED); multiples of 128
 *                    copy twice as many keys per TMA transfer.
 *   cu_seqlens_q     NULL for decode (one query per sequence, n_q_rows ==
 *                    batch), else as for mla_attn_prefill_chunk (then
 *                    num_splits must be 0 or 1).
 *   max_seqlen_k     host upper bound of the key counts (plans the splits).
 *   o_lat            [n_q_rows, H, C] written.
 *   workspace        at least mla_workspace_size(dims, batch, n_q_rows,
 *                    max_seqlen_k, num_splits) bytes.
 * num_pages * page_size must stay below 2^31 for the tensor-core kernels. */
MLA_API mla_status_t mla_attn_paged(const mla_dims_t* dims, const void* q_abs, const void* q, int64_t q_row_stride,
                                    const int32_t* cu_seqlens_q, int64_t n_q_rows, const int32_t* seqlens_k,
                                    int32_t batch, int64_t max_seqlen_k, const void* kv_cache,
                                    const void* pe_cache, int64_t num_pages, int32_t page_size,
                                    const int32_t* block_table, int64_t max_pages_per_seq, void* o_lat,
                                    void* workspace, size_t workspace_bytes, int32_t num_splits,
                                    cudaStream_t stream);

/* Bytes of workspace mla_attn_sparse_decode needs (num_splits as for
 * mla_attn_decode; 0 = automatic).  0 for dims the call does not support. */
MLA_API size_t mla_sparse_workspace_size(const mla_dims_t* dims, int32_t batch, int32_t max_topk,
                                         int32_t num_splits);

/* Token-granular sparse decode: one query per sequence attends to a selected
 * list of cache rows only ("What is DeepSeek Sparse Attention (DSA)? A clear,
 * modern explainer", section "How DSA works (conceptual)": exact attention
 * over the shortlisted tokens).  The selector itself is not part of the call.
 *   indices      device int32 [batch, index_stride]: row b lists the cache rows
 *                (of kv_cache / pe_cache, any rows, any order) sequence b
 *                attends to; a row listed twice counts twice.
 *   counts       device int32 [batch]: entries of row b that are used (clamped
 *                to 0 .. max_topk); entries past them are never read.  A used
 *                entry outside [0, kv_rows) reads as a key of zeros and sets
 *                bit 1<<7 of the device error word.
 *   max_topk     host upper bound of the counts; index_stride >= max_topk.
 *   batch        at most 65535.
 *   q_abs, q, q_row_stride, kv_cache, pe_cache, kv_rows, o_lat [batch, H, C],
 *   num_splits   as for mla_attn_decode.
 *   workspace    at least mla_sparse_workspace_size(dims, batch, max_topk,
 *                num_splits) bytes, 16-byte aligned.  The call copies the
 *                selected rows there (one page per sequence) and runs the
 *                paged attention (mla_attn_paged) over them.
 * Needs C and R rows of a multiple of 16 bytes (C <= 512 bf16 / 256 fp32
 * values, R <= 256 / 128); other dims return MLA_ERR_UNSUPPORTED. */
MLA_API mla_status_t mla_attn_sparse_decode(const mla_dims_t* dims, const void* q_abs, const void* q,
                                            int64_t q_row_stride, const void* kv_cache, const void* pe_cache,
                                            int64_t kv_rows, const int32_t* indices, int64_t index_stride,
                                            const int32_t* counts, int32_t batch, int32_t max_topk, void* o_lat,
                                            void* workspace, size_t workspace_bytes, int32_t num_splits,
                                            cudaStream_t stream);

/* Output projection: out[n,h,d] = sum_c o_lat[n,h,c] * wkv_b[h*(Dn+Dv)+Dn+d, c].
 * ("Absorb Path Execution", the last einsum, with the tail rows of wkv_b.)
 *   o_lat [n_rows, H, C] contiguous; out [n_rows, H, Dv] contiguous, written.
 *   The tensor-core kernel takes at most 65535 * 256 rows per call.
 * The tensor-core kernel may start while the previous kernel on the stream is
 * still finishing (programmatic dependent launch, when that kernel allows it,
 * as this library's attention calls do) and reads wkv_b before waiting for it:
 * wkv_b must not be written by a kernel that allows its successor to start
 * early.  o_lat is read only after the previous kernel has completed. */
MLA_API mla_status_t mla_out_proj(const mla_dims_t* dims, const void* o_lat, const void* wkv_b, void* out,
                          int64_t n_rows, cudaStream_t stream);

/* Latent KV expansion, the naive path's materialisation ("Latent KV expansion
 * with split", the operation's description; its output is the per-head keys
 * and values "Naive Path Execution" consumes):
 *   x[t]               = kv_c[t] / sqrt(mean_c(kv_c[t]^2) + eps) * gamma
 *   k_nope[b, h, s, d] = sum_c x[b*S+s, c] * wkv_b[h*(Dn+Dv) + d, c]        d < Dn
 *   v[b, h, s, d]      = sum_c x[b*S+s, c] * wkv_b[h*(Dn+Dv) + Dn + d, c]   d < Dv
 *   kv_c    [batch * seq_len, C] row-major (compressed KV before normalisation;
 *           packed tokens of ragged sequences may pass batch = 1).
 *   gamma   [C] RMSNorm gain, or NULL for 1.   eps >= 0.
 *   wkv_b   [H*(Dn+Dv), C] row-major.
 *   k_nope  [batch, H, seq_len, Dn] and v [batch, H, seq_len, Dv], written.
 * bf16 DeepSeek-V3 shapes run on the tcgen05 kernel (the normalised row is
 * rounded to bf16 after the gain, the row's RMS factor scales the fp32
 * products); other shapes on a CUDA-core kernel. */
MLA_API mla_status_t mla_expand_kv(const mla_dims_t* dims, const void* kv_c, const void* gamma, float eps,
                                   const void* wkv_b, int64_t batch, int64_t seq_len, void* k_nope, void* v,
                                   cudaStream_t stream);

/* Append new tokens to the latent caches ("Absorb Implementation Cache Design":
 * kv_cache holds the compressed key-value vector, pe_cache the rotary key;
 * "Latent KV expansion with split": the compressed KV is RMS-normalised):
 *   kv_cache[slots[n], c] = kv_new[n, c] / sqrt(mean_c(kv_new[n]^2) + eps) * gamma[c]
 *   pe_cache[slots[n], 2i]   = a cos t - b sin t      (a, b) = k_pe_new[n, 2i], k_pe_new[n, 2i+1]
 *   pe_cache[slots[n], 2i+1] = a sin t + b cos t      t = positions[n] * rope_base^(-2i/R)
 *   kv_new      [n_tokens, C], k_pe_new [n_tokens, R] (before normalisation / rotation).
 *   gamma       [C] RMSNorm gain, or NULL for 1.
 *   eps         >= 0; rope_base > 0 (10000 for DeepSeek-V3).
 *   positions   device int32 [n_tokens]: the token's index in its sequence.
 *   slots       device int64 [n_tokens]: destination row of both caches; a slot
 *               outside [0, cache_rows) is skipped.  Slots must be distinct.
 *   kv_cache    [cache_rows, C], pe_cache [cache_rows, R], updated in place.
 * Needs C a multiple of 8 (bf16) or 4 (fp32), C <= 1024, R even, R <= 128;
 * other dims return MLA_ERR_UNSUPPORTED. */
MLA_API mla_status_t mla_append_latent(const mla_dims_t* dims, const void* kv_new, const void* k_pe_new,
                                       const void* gamma, float eps, float rope_base, const int32_t* positions,
                                       const int64_t* slots, int64_t n_tokens, void* kv_cache, void* pe_cache,
                                       int64_t cache_rows, cudaStream_t stream);

/* Static text for a status code. */
MLA_API const char* mla_status_string(mla_status_t status);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device.  Returns MLA_ERR_DEVICE_TIMEOUT if an earlier kernel set a
 * bit of the word (stored in *code_out when non-NULL), MLA_ERR_CUDA if the
 * stream reports an error, MLA_OK otherwise.  Bits: 1<<0 a consumer waited too
 * long for a TMA tile, 1<<1 a producer for a free stage, 1<<2 a wait for a
 * tensor-core commit, 1<<3 a wait on the softmax threads (P, q_abs in TMEM), 1<<4 a wait on the partner
 * CTA, 1<<5 an exit path for copies in flight, 1<<6 a work item outside its
 * buffers (or a misaligned shared-memory base), 1<<7 a block-table entry of a
 * page that holds keys lies outside the cache (mla_attn_paged). */
MLA_API mla_status_t mla_device_status(cudaStream_t stream, uint32_t* code_out);

/* Which kernel family a call with these dims runs: 1 = tcgen05 tensor-core
 * kernels, 0 = CUDA-core kernels, -1 = unsupported dims. */
MLA_API int32_t mla_kernel_family(const mla_dims_t* dims);

/* MLA_API_VERSION of the built library. */
MLA_API int32_t mla_api_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H_ */
