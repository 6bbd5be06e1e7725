/*
 * cpattn.h -- C ABI of libcpattn.so, the B200 (sm_100a) hot path of
 * context-parallel attention emulated on one GPU.
 *
 * Sources (web pages, cited by title and section):
 *   [CP]  diffusers v0.43.0 docs, "Context parallelism": variants table;
 *         "Ring Attention"; "Ulysses Attention"; "Unified Attention";
 *         "Ulysses Anything Attention"; "Ring Anything Attention".
 *   [SP]  SGLang Diffusion docs, "Sequence Parallelism": "Choosing The
 *         Attention Exchange"; "Numerics across node boundaries".
 *   [USP] "Ulysses Sequence Parallelism: training with million-token
 *         contexts": sections 3 (core idea), 4 (steps), 5 (communication),
 *         7 (causal masking by position ids).
 *   [API] diffusers docs, "parallel": ContextParallelConfig parameters
 *         ring_degree, ulysses_degree, convert_to_fp32, rotate_method,
 *         ulysses_anything, ring_anything.
 *   [PR]  sglang PR #30086 analysis: (B, S, H, D) q/k/v view, scale
 *         head_dim**-0.5.
 *
 * Conventions for every entry point
 * ---------------------------------
 * Tensors.  Q, K, V and attention outputs are bf16, (batch B, seq S, heads H,
 *   head_dim D) contiguous ("BSHD", [PR]).  D must be 64 or 128.  Softmax
 *   scale is D**-0.5 ([PR]).  Attention is non-causal with no mask ([SP]
 *   kv_gather constraint; [CP] Ring Anything requires attn_mask None), except
 *   in the cpattn_causal_* entry points (section "causal" below).
 *   LSE outputs are float32, natural log, layout (B, H, S).
 * Shards.  A "sequence shard" r of a full BSHD tensor is rows off_r ..
 *   off_r + len_r - 1 of every batch element, with off_r the prefix sum of the
 *   lengths.  NULL length arrays mean the standard equal split, which requires
 *   divisibility by the degree ([CP] variants table); explicit lengths are the
 *   'anything' modes ([CP] Ring Anything / Ulysses Anything), may be uneven and
 *   may contain zeros.
 * Contexts.  The library keeps per-device state for the life of the process
 *   (kernel attributes set on first use, cluster sizes, the no-allocation
 *   scratch address): use it under each device's primary context, the one the
 *   CUDA runtime uses, and not across a cudaDeviceReset.  An entry point
 *   called on a thread that has no context current yet (a worker thread that
 *   made no CUDA call) binds the current device's primary context to that
 *   thread (cudaSetDevice) before it encodes any tensor map.
 * Memory.  All tensor pointers are DEVICE pointers owned by the caller; the
 *   library allocates no device memory on any call (workspaces come from the
 *   caller; cpattn_ulysses_attention_noalloc uses a static scratch).  Length/split arrays are HOST arrays read only
 *   during the call.  Q, K, V and outputs must be 16-byte aligned.  Outputs
 *   must not alias inputs unless stated.
 * Streams.  `stream` is a cudaStream_t (NULL = legacy default stream).  Every
 *   call only enqueues work; none synchronises the host.  Arguments are fully
 *   validated before anything is enqueued; on a non-zero return nothing was
 *   enqueued except for CPATTN_ERR_CUDA, which reports a launch failure.
 *   The compute calls can be captured in a CUDA graph (after one eager call
 *   per kernel shape, which sets the kernels' shared-memory attribute and,
 *   for the projections, sizes their two-CTA cluster grid): nothing on their
 *   launch path synchronises or allocates, and each launch carries its plan
 *   by value.  cpattn_device_status synchronises and is not
 *   capturable.
 * Errors.  Return value is a cpattn_status.  No C++ exception crosses the ABI.
 *   Device-side bounded waits (see cpattn_device_status) report a pipeline that
 *   stopped making progress instead of hanging the GPU.
 */
#ifndef CPATTN_H
#define CPATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *cpattn_stream_t; /* == cudaStream_t */

typedef enum {
  CPATTN_OK = 0,
  CPATTN_ERR_NULL = 1,           /* a required pointer is NULL                        */
  CPATTN_ERR_SHAPE = 2,          /* B, H, S < 1, D not 64/128, elem size unsupported  */
  CPATTN_ERR_INDIVISIBLE = 3,    /* lengths NULL and S or H not divisible by degree   */
  CPATTN_ERR_SPLITS = 4,         /* negative lengths or lengths not summing to S / H  */
  CPATTN_ERR_DEGREE = 5,         /* degree < 1, degree > S (or > H), step out of range */
  CPATTN_ERR_CUDA = 6,           /* CUDA runtime/driver error (no device, launch)     */
  CPATTN_ERR_DEVICE_TIMEOUT = 7, /* a device-side bounded wait expired                */
  CPATTN_ERR_WORKSPACE = 8,      /* workspace NULL or smaller than required           */
  CPATTN_ERR_ALIGNMENT = 9,      /* a tensor pointer is not 16-byte aligned           */
  CPATTN_ERR_UNSUPPORTED = 10    /* current device is not sm_100 (B200)               */
} cpattn_status;

/* Human-readable name of a status code; never NULL. */
const char *cpattn_status_string(int status);

/*
 * The CUDA error behind the last CPATTN_ERR_CUDA returned on the calling
 * thread (a cudaError_t value; 0 if none was recorded), and a description of
 * it, "<step>: <error name> (<error string>)", where <step> names what failed
 * (a kernel launch, a device query, a tensor-map encoding, ...).  The string
 * is thread-local and stays valid until the thread's next call of this
 * function; never NULL.  Neither call touches the device.
 */
int cpattn_last_cuda_error(void);
const char *cpattn_last_cuda_error_string(void);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int cpattn_version(void);

/* ------------------------------------------------------------------ ring */

/*
 * Ring attention, fused ([CP] "Ring Attention", "Ring Anything Attention";
 * [API] ring_degree, convert_to_fp32, rotate_method).
 *
 * The sequence is cut into `ring_degree` shards; rank r holds shard r of Q, K
 * and V.  For every rank the kernel walks the K/V chunks in ring order
 * c = r, r-1, ..., r-P+1 (mod P) -- the block a GPU holds after t hand-offs --
 * computing the attention of Q shard r against one chunk at a time and merging
 * it into a running float32 (out, LSE) state with the online-softmax / LSE
 * rule, so that after the full ring every query has seen every key.  The merge
 * is held on chip (TMEM/registers) instead of in HBM; cpattn_ring_step +
 * cpattn_lse_merge is the same computation with the partials in memory.
 *
 *   q, k, v    [B, S, H, D] bf16 device, read only.
 *   out        [B, S, H, D] bf16 device, written (all rows).
 *   lse        [B, H, S] float32 device, natural log; may be NULL.
 *   chunk_lens host int[ring_degree] (Ring Anything) or NULL (equal split,
 *              S % ring_degree must be 0 else CPATTN_ERR_INDIVISIBLE).
 * Errors: NULL, SHAPE, DEGREE (ring_degree < 1, > S, or > 512), INDIVISIBLE, SPLITS,
 * ALIGNMENT, UNSUPPORTED, CUDA.
 */
int cpattn_ring_attention(const void *q, const void *k, const void *v, void *out, float *lse,
                          int B, int H, int S, int D, int ring_degree, const int *chunk_lens,
                          cpattn_stream_t stream);

/*
 * One ring step for every rank ([CP] "Ring Attention"; [API] convert_to_fp32):
 * rank r attends its Q shard to chunk c = (r - step) mod P and writes the
 * partial result normalised over that chunk, in float32, plus its LSE.
 * A rank whose chunk is empty writes out = 0 and LSE = -inf for its rows.
 *
 *   part_out   [B, S, H, D] float32 device (rows of shard r hold rank r's partial).
 *   part_lse   [B, H, S] float32 device.
 *   step       0 <= step < ring_degree (else CPATTN_ERR_DEGREE).
 * Other arguments as cpattn_ring_attention.
 */
int cpattn_ring_step(const void *q, const void *k, const void *v, float *part_out,
                     float *part_lse, int B, int H, int S, int D, int ring_degree,
                     const int *chunk_lens, int step, cpattn_stream_t stream);

/*
 * LSE merge of P float32 partials ([SP] "Numerics across node boundaries":
 * online-softmax merge of the ring's partial results; [API] convert_to_fp32):
 *   M = max_p LSE_p,  LSE = M + ln sum_p exp(LSE_p - M),
 *   out = sum_p exp(LSE_p - LSE) * out_p.
 * Partials with LSE = -inf carry no keys and get weight 0; rows where every
 * partial is empty produce out = 0, LSE = -inf.
 *
 *   part_out   P consecutive [B, S, H, D] float32 tensors (device).
 *   part_lse   P consecutive [B, H, S] float32 tensors (device).
 *   out_f32    [B, S, H, D] float32 or NULL.  May alias part_out (partial 0):
 *              each element is read before it is written, by the same thread.
 *   out_bf16   [B, S, H, D] bf16 or NULL.  At least one of out_f32/out_bf16.
 *   lse_out    [B, H, S] float32 or NULL.  May alias part_lse (partial 0).
 * Errors: NULL, SHAPE (P < 1), ALIGNMENT, CUDA.
 */
int cpattn_lse_merge(const float *part_out, const float *part_lse, int P, int B, int H, int S,
                     int D, float *out_f32, void *out_bf16, float *lse_out,
                     cpattn_stream_t stream);

/* ------------------------------------------------------------- kv_gather */

/*
 * kv_gather exchange ([SP] "Choosing The Attention Exchange"): Q and the
 * output stay sequence-sharded, K and V are gathered in full (on one GPU they
 * already are), and every rank computes the attention of its own Q rows
 * against all S keys; non-causal, ring degree 1.
 *
 *   q_lens     host int[degree] or NULL (equal split).
 * Other arguments as cpattn_ring_attention; degree may be up to 1024.
 */
int cpattn_kv_gather_attention(const void *q, const void *k, const void *v, void *out,
                               float *lse, int B, int H, int S, int D, int degree,
                               const int *q_lens, cpattn_stream_t stream);

/* --------------------------------------------------------------- Ulysses */

/*
 * Ulysses permute, sequence-sharded -> head-sharded: the first all-to-all
 * ([CP] "Ulysses Attention": every GPU ends up with every token for a subset
 * of the heads; [USP] section 4), with uneven splits ([CP] "Ulysses Anything
 * Attention"):
 *     y_{r'}[b, s, h - hoff_{r'}, :] = x_{r(s)}[b, s - off_{r(s)}, h, :]
 *
 *   x  sequence side: the `degree` rank buffers concatenated in rank order,
 *      rank r = [B, seq_r, H, D] (for B = 1 this is the full [1, S, H, D]).
 *   y  head side: the rank buffers concatenated in rank order,
 *      rank r' = [B, S, head_r', D].
 *   elem_bytes  element size (2 for bf16 Q/K/V, 4 for float32); D*elem_bytes
 *      must be a multiple of 16.  Data is moved bit-exactly.
 *   seq_splits / head_splits  host int[degree] or NULL (equal split; S and H
 *      must then be divisible by degree, else CPATTN_ERR_INDIVISIBLE).
 * x and y must not overlap.  Errors: NULL, SHAPE, DEGREE (degree < 1),
 * INDIVISIBLE, SPLITS, ALIGNMENT, CUDA.
 */
int cpattn_ulysses_permute(const void *x, void *y, int B, int S, int H, int D, int elem_bytes,
                           int degree, const int *seq_splits, const int *head_splits,
                           cpattn_stream_t stream);

/*
 * The first all-to-all of the Ulysses flow for Q, K and V at once: the
 * cpattn_ulysses_permute of each of the three tensors (same shape, element
 * size and splits), in one launch.  q, k, v are read, yq, yk, yv written; the
 * six buffers must not alias.  Arguments and errors as cpattn_ulysses_permute.
 */
int cpattn_ulysses_permute_qkv(const void *q, const void *k, const void *v, void *yq, void *yk,
                               void *yv, int B, int S, int H, int D, int elem_bytes, int degree,
                               const int *seq_splits, const int *head_splits,
                               cpattn_stream_t stream);

/*
 * Ulysses unpermute, head-sharded -> sequence-sharded: the second all-to-all,
 * which regroups the attention output by token ([CP] "Ulysses Attention");
 * the exact inverse of cpattn_ulysses_permute (same arguments, y is read and
 * x is written).
 */
int cpattn_ulysses_unpermute(const void *y, void *x, int B, int S, int H, int D, int elem_bytes,
                             int degree, const int *seq_splits, const int *head_splits,
                             cpattn_stream_t stream);

/*
 * The Ulysses projections with the all-to-alls fused in ([USP] section 4: each
 * rank projects its sequence chunk to Q, K and V, the first all-to-all
 * regroups them by head, and after local attention and the second all-to-all
 * each rank applies the output projection to its chunk).
 *
 * cpattn_ulysses_qkv_projection: for every sequence rank r,
 *     QKV_r = X_r W_qkv^T   (bf16 in, fp32 accumulate, rounded to bf16),
 * split into Q | K | V, each (B, S_r, H, D), and stored directly in the
 * head-sharded layout: the result equals cpattn_ulysses_permute_qkv applied
 * to the three unfused projections, with no intermediate tensor.
 *   x          sequence side: rank buffers (B, S_r, Dm) concatenated in rank
 *              order, bf16 (for B = 1 the plain (S, Dm) activations).
 *   w_qkv      (3*H*D, Dm) bf16 row-major (the nn.Linear weight layout):
 *              rows [t*H*D + h*D, t*H*D + (h+1)*D) are head h of Q (t = 0),
 *              K (t = 1) or V (t = 2).
 *   yq, yk, yv head side: rank buffers (B, S, H_u, D) concatenated, bf16.
 *   Dm         model width, a positive multiple of 64.  D is 64 or 128.
 *   degree, seq_splits, head_splits as cpattn_ulysses_permute.
 * No bias is added.
 *
 * cpattn_ulysses_output_projection: the second all-to-all fused into the
 * output projection.  For every sequence rank r,
 *     out_r = O_r W_o^T,  O_r = the rank's tokens of every head, (B, S_r, H*D),
 * where O_r is read straight from the head-sharded attention output yo (the
 * result equals cpattn_ulysses_unpermute followed by the projection).
 *   yo         head side, as yq above (bf16).
 *   w_o        (Dm, H*D) bf16 row-major.
 *   out        sequence side: rank buffers (B, S_r, Dm) concatenated, bf16.
 *
 * All pointers are device memory owned by the caller, 16-byte aligned; inputs
 * and outputs must not alias.  Errors: CPATTN_ERR_NULL, CPATTN_ERR_SHAPE (B, S,
 * H < 1, D not 64/128, Dm not a positive multiple of 64, H > 1024),
 * CPATTN_ERR_DEGREE (degree outside 1..64), CPATTN_ERR_INDIVISIBLE,
 * CPATTN_ERR_SPLITS, CPATTN_ERR_ALIGNMENT, CPATTN_ERR_UNSUPPORTED,
 * CPATTN_ERR_CUDA; nothing is launched on an error.
 */
int cpattn_ulysses_qkv_projection(const void *x, const void *w_qkv, void *yq, void *yk, void *yv,
                                  int B, int S, int H, int D, int Dm, int degree,
                                  const int *seq_splits, const int *head_splits,
                                  cpattn_stream_t stream);
int cpattn_ulysses_output_projection(const void *yo, const void *w_o, void *out, int B, int S,
                                     int H, int D, int Dm, int degree, const int *seq_splits,
                                     const int *head_splits, cpattn_stream_t stream);

/*
 * Head-sharded local attention ([USP] section 4: after the first all-to-all
 * every GPU runs ordinary attention over all tokens of its heads): for every
 * head rank r', attention of its [B, S, head_r', D] Q/K/V buffers.
 *
 *   yq, yk, yv, yo  head-sharded layouts as in cpattn_ulysses_permute (bf16).
 *   lse        [B, H, S] float32 indexed by global head, or NULL.
 */
int cpattn_head_sharded_attention(const void *yq, const void *yk, const void *yv, void *yo,
                                  float *lse, int B, int H, int S, int D, int degree,
                                  const int *head_splits, cpattn_stream_t stream);

/* Bytes of workspace cpattn_ulysses_attention needs: 4 * B*S*H*D * 2. */
size_t cpattn_ulysses_workspace_bytes(int B, int H, int S, int D);

/*
 * Ulysses attention ([CP] "Ulysses Attention"; [USP] section 4): permute Q, K,
 * V to the head-sharded layout (one launch), then local attention per head
 * rank whose epilogue stores every output row straight into the
 * sequence-sharded layout -- the second all-to-all, fused into the attention
 * kernel (one launch).  q, k, v, out are sequence-side rank buffers as `x` in
 * cpattn_ulysses_permute; lse is [B, H, S] (global head and token) or NULL.
 * workspace: device, >= cpattn_ulysses_workspace_bytes, 16-byte aligned,
 * caller-owned scratch (contents undefined after the call).
 */
int cpattn_ulysses_attention(const void *q, const void *k, const void *v, void *out, float *lse,
                             int B, int H, int S, int D, int degree, const int *seq_splits,
                             const int *head_splits, void *workspace, size_t workspace_bytes,
                             cpattn_stream_t stream);

/* --------------------------------------------------------------- unified */

/* Bytes of workspace cpattn_unified_attention needs: 4 * B*S*H*D * 2. */
size_t cpattn_unified_workspace_bytes(int B, int H, int S, int D);

/*
 * Unified ring x Ulysses attention ([CP] "Unified Attention": an all-to-all
 * redistributes heads and tokens, ring attention runs on the result, and the
 * inverse all-to-all restores the layout; the GPUs form a
 * ring_degree x ulysses_degree grid).
 *
 * Ring chunks are the outer split of the sequence (ring_lens, or equal);
 * inside ring chunk i the ulysses_degree ranks of that Ulysses group hold
 * sub-shards of it; heads are split by head_splits (or equally).  Steps: per
 * ring group, Ulysses permute of its chunk to head groups (one launch for all
 * groups); per head group, ring attention over the chunks with the LSE merge,
 * whose epilogue stores the output at its token and global head in `out` --
 * the inverse permute, fused (one launch).
 *
 *   q, k, v, out  full [B, S, H, D] bf16.  lse [B, H, S] or NULL.
 *   ring_lens     host int[ring_degree] or NULL (equal split).
 *   head_splits   host int[ulysses_degree] or NULL (equal split).
 *   workspace     >= cpattn_unified_workspace_bytes.
 */
int cpattn_unified_attention(const void *q, const void *k, const void *v, void *out, float *lse,
                             int B, int H, int S, int D, int ring_degree, int ulysses_degree,
                             const int *ring_lens, const int *head_splits, void *workspace,
                             size_t workspace_bytes, cpattn_stream_t stream);

/* ------------------------------------- building blocks of the exchanges */

/*
 * The calls below are what one rank runs when the shards live on different
 * GPUs and the exchanges are real collectives (the Python module
 * context_attention_long_b200.exchange moves the data with torch.distributed
 * over NCCL and calls these for every step of local compute).
 */

/*
 * One ring step of one rank, merged into the rank's running result
 * ([CP] "Ring Attention": each GPU computes attention against the K/V block it
 * holds, then passes the block on; [API] convert_to_fp32: the partial output
 * and its LSE are kept in float32; [SP] "Numerics across node boundaries":
 * partial results are combined with the online-softmax merge; [SP]
 * "Cross-Node Sequence Parallelism": the point-to-point rotation overlaps the
 * attention of the block already held).
 *
 * Attention of the rank's queries against the one K/V chunk it holds now:
 *   q          [B, Sq, H, D] bf16, sequence positions q_pos0 .. q_pos0+Sq-1.
 *   k, v       [B, kv_batch_rows, H, D] bf16; the first Skv rows of every
 *              batch element are the chunk (positions kv_pos0 ..);
 *              kv_batch_rows = Skv for a contiguous chunk, larger for a chunk
 *              padded to the longest one (the all-gather of [CP] "Ring
 *              Anything Attention").  Skv may be 0 (an empty chunk).
 *   prev_out   NULL: no earlier state; out and lse receive this chunk's
 *              partial result (normalised over its keys) and its LSE.
 *              Otherwise float32 [B, Sq, H, D], the running result over the
 *              chunks already visited, whose LSE is in `lse` on entry; out and
 *              lse receive the LSE-rule merge of the two.  May alias out when
 *              out_f32 = 1 (each element is read before it is written, by the
 *              same thread).
 *   out        [B, Sq, H, D], float32 (out_f32 = 1: an intermediate state) or
 *              bf16 (out_f32 = 0: the final output).
 *   lse        [B, H, Sq] float32, natural log; required (see prev_out).
 *   causal     1: key j is visible to query i iff kv_pos0 + j <= q_pos0 + i
 *              ([USP] section 7: masking by positions).  A query that sees no
 *              key of the chunk keeps the earlier state unchanged (out = 0 and
 *              LSE = -inf without one).
 * Errors: NULL, SHAPE (B, H, Sq < 1, Skv < 0, kv_batch_rows < max(Skv, 1),
 * negative positions, D not 64/128), ALIGNMENT, UNSUPPORTED, CUDA.
 */
int cpattn_ring_chunk_attention(const void *q, const void *k, const void *v, void *out, float *lse,
                                const float *prev_out, int B, int H, int Sq, int Skv, int kv_batch_rows, int D,
                                int q_pos0, int kv_pos0, int causal, int out_f32, cpattn_stream_t stream);

/*
 * Attention of one rank's query shard against K/V chunks gathered from every
 * rank ([SP] "Choosing The Attention Exchange": kv_gather all-gathers K and V
 * and each rank computes its own rows; [API] rotate_method "allgather": ring
 * attention gathers the chunks, then walks them; [CP] "Ring Anything
 * Attention": chunks are padded to the longest before the all-gather and
 * sliced back before attention).  One launch; the chunks are visited in ring
 * order from the rank's own chunk with the running (m, l, O) state on chip.
 *
 *   k, v       `degree` consecutive [B, kv_batch_rows, H, D] bf16 blocks
 *              (what an all-gather of padded chunks delivers); chunk c holds
 *              kv_lens[c] <= kv_batch_rows valid rows per batch element, at
 *              sequence positions off_c = kv_lens[0] + ... + kv_lens[c-1].
 *   kv_lens    host int[degree], zeros allowed; NULL: every chunk has
 *              kv_batch_rows rows.
 *   rank       0 <= rank < degree: the shard the queries belong to.
 *   q, out     [B, kv_lens[rank], H, D] bf16, the rank's own tokens.
 *   lse        [B, H, kv_lens[rank]] float32 or NULL.
 *   causal     1: chunks after `rank` are skipped and the own chunk is masked
 *              by position (the ring's use; kv_gather itself is non-causal).
 * Errors: NULL, SHAPE (kv_lens[rank] = 0 included), DEGREE (degree outside
 * 1..512, rank outside 0..degree-1), SPLITS (a length < 0 or >
 * kv_batch_rows), ALIGNMENT, UNSUPPORTED, CUDA.
 */
int cpattn_gathered_kv_attention(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
                                 int D, int degree, const int *kv_lens, int kv_batch_rows, int rank, int causal,
                                 cpattn_stream_t stream);

/*
 * Attention over a sequence held as `degree` rank buffers [B, S_u, H, D]
 * concatenated in rank order -- the layout in which the first all-to-all of
 * Ulysses attention delivers a rank's heads ([CP] "Ulysses Attention";
 * [USP] section 4: after the all-to-all every GPU holds every token of a
 * subset of the heads and runs ordinary attention over them).  Every query
 * attends all S keys of its batch element (causal = 1: the keys at
 * positions <= its own, a token's position being its index in the full
 * sequence); the output is written in the same layout, ready for the second
 * all-to-all.
 *
 *   q, k, v, out  rank-buffer layout, bf16 (for B = 1 the plain [1, S, H, D]).
 *   lse           [B, H, S] float32 (global positions) or NULL.
 *   seq_splits    host int[degree] or NULL (equal split).
 * Errors: NULL, SHAPE, DEGREE (degree outside 1..64), INDIVISIBLE, SPLITS,
 * ALIGNMENT, UNSUPPORTED, CUDA.
 */
int cpattn_rank_buffer_attention(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
                                 int S, int D, int degree, const int *seq_splits, int causal,
                                 cpattn_stream_t stream);

/* ---------------------------------------------------------------- causal */

/*
 * Causal variants ([USP] section 7: for causal masking over long sequences,
 * Ulysses and ring attention use position ids instead of an attention-mask
 * tensor).  Every token's position is its index s in the full sequence; key
 * j is visible to query i iff j <= i.  No mask tensor exists: the kernel
 * derives the mask from the positions of the row ranges it walks, skips every
 * K/V tile that lies wholly after a Q tile's last query, and masks inside the
 * tiles that straddle the diagonal.  The kv_gather exchange has no causal
 * variant ([SP] "Choosing The Attention Exchange": kv_gather is non-causal).
 *
 * Each function takes exactly the arguments, layouts, ownership and error
 * behaviour of its non-causal namesake:
 *   cpattn_causal_ring_attention        as cpattn_ring_attention.  Rank r
 *       walks the chunks before its shard in ring order (r-1, ..., 0) and its
 *       own chunk, the one the mask cuts, last; chunks after shard r are
 *       invisible to all of its queries and are not visited.  The merge is
 *       order-independent in exact arithmetic.
 *   cpattn_causal_ring_step             as cpattn_ring_step.  A step whose
 *       chunk lies after shard r writes out = 0 and LSE = -inf for its rows
 *       (the neutral partial), so cpattn_lse_merge of all steps equals
 *       cpattn_causal_ring_attention.
 *   cpattn_causal_head_sharded_attention as cpattn_head_sharded_attention
 *       (positions 0 .. S-1 in every head-side buffer).
 *   cpattn_causal_ulysses_attention     as cpattn_ulysses_attention.
 *   cpattn_causal_unified_attention     as cpattn_unified_attention (ring
 *       chunk i holds positions off_i .. off_i + len_i - 1).
 */
int cpattn_causal_ring_attention(const void *q, const void *k, const void *v, void *out, float *lse,
                                 int B, int H, int S, int D, int ring_degree,
                                 const int *chunk_lens, cpattn_stream_t stream);
int cpattn_causal_ring_step(const void *q, const void *k, const void *v, float *part_out,
                            float *part_lse, int B, int H, int S, int D, int ring_degree,
                            const int *chunk_lens, int step, cpattn_stream_t stream);
int cpattn_causal_head_sharded_attention(const void *yq, const void *yk, const void *yv, void *yo,
                                         float *lse, int B, int H, int S, int D, int degree,
                                         const int *head_splits, cpattn_stream_t stream);
int cpattn_causal_ulysses_attention(const void *q, const void *k, const void *v, void *out,
                                    float *lse, int B, int H, int S, int D, int degree,
                                    const int *seq_splits, const int *head_splits, void *workspace,
                                    size_t workspace_bytes, cpattn_stream_t stream);
int cpattn_causal_unified_attention(const void *q, const void *k, const void *v, void *out,
                                    float *lse, int B, int H, int S, int D, int ring_degree,
                                    int ulysses_degree, const int *ring_lens, const int *head_splits,
                                    void *workspace, size_t workspace_bytes, cpattn_stream_t stream);

/* -------------------------------------------------------------- backward */

/*
 * Gradient of attention with respect to Q, K and V, for training over long
 * contexts ([USP] sections 1 and 7).  It is the derivative of the forward
 * definition; the pages print no backward formulas.  Per (batch, head), with
 * S = Q K^T * D**-0.5, P = softmax(S) recomputed from the forward's LSE, and
 * dO the upstream gradient of the output O:
 *   dV = P^T dO,  dS = P * (dO V^T - rowsum(dO * O)),
 *   dQ = dS K * D**-0.5,  dK = dS^T Q * D**-0.5.
 * The ring, Ulysses and unified paths compute this same attention, so this is
 * their gradient too; causal = 1 applies the cpattn_causal_* mask (key j
 * visible to query i iff j <= i).
 *
 *   q, k, v, out, dout  [B, S, H, D] bf16 device, read only (out: the forward
 *                       output; dout: the gradient of the loss with respect
 *                       to it).
 *   lse                 [B, H, S] float32 device, natural log (the forward's).
 *   dq, dk, dv          [B, S, H, D] bf16 device, written.
 *   workspace           device, at least
 *                       cpattn_attention_backward_workspace_bytes(B, H, S)
 *                       bytes, 4-byte aligned (holds rowsum(dO * O)).  Bytes
 *                       beyond that, from the next 256-byte boundary, are
 *                       scratch for dS: each head takes
 *                       cpattn_attention_backward_ds_bytes(B, S, causal).
 * With scratch for at least one head: the row sums, then per group of heads
 * whose dS fits the scratch together (all heads in one group when it holds
 * H heads' worth) a dK/dV kernel (one CTA per K/V tile, walking the Q tiles)
 * that also stores dS in bf16, and a dQ GEMM (dQ = dS K * D**-0.5, persistent,
 * reading the stored dS).  Without: the row sums, a dQ kernel (one CTA per Q
 * tile, walking the K/V tiles and computing S and dP again) and the dK/dV
 * kernel.  No atomics either way, and dK and dV are the same bytes in both;
 * dQ differs by the rounding of the dS the two kernels form.  Errors: NULL,
 * SHAPE (also when B*S*H >= 2^31, a tensor larger than any device memory),
 * WORKSPACE, ALIGNMENT, UNSUPPORTED, CUDA.
 */
size_t cpattn_attention_backward_workspace_bytes(int B, int H, int S);
/* Bytes of dS scratch one head takes: B * 32 KB per (Q tile, K tile) pair of
 * 128-row tiles, all pairs, or under the causal mask (causal != 0) those with
 * the K tile at or before the Q tile.  0 when B or S < 1. */
size_t cpattn_attention_backward_ds_bytes(int B, int S, int causal);
int cpattn_attention_backward(const void *q, const void *k, const void *v, const void *out,
                              const float *lse, const void *dout, void *dq, void *dk, void *dv,
                              int B, int H, int S, int D, int causal, void *workspace,
                              size_t workspace_bytes, cpattn_stream_t stream);

/*
 * Backward of the Ulysses flow ([USP] section 4 run in reverse for training,
 * sections 1 and 7): the first all-to-all takes Q, K, V, the forward output O
 * and its gradient dO to the head-sharded layout (two launches), and the
 * attention backward of cpattn_attention_backward runs on every head rank's
 * buffers (its kernels cover up to 8 head ranks, or groups of heads, per
 * launch).  The second all-to-all is fused: the kernels store dQ, dK and dV
 * straight into the sequence-sharded rank buffers.
 *
 *   q, k, v, out, dout  sequence-sharded rank buffers, as the inputs and the
 *                       output of cpattn_ulysses_attention; read only.
 *   lse                 [B, H, S] float32 device, from the forward.
 *   dq, dk, dv          sequence-sharded rank buffers, written.
 *   workspace           device, 16-byte aligned, at least
 *                       cpattn_ulysses_attention_backward_workspace_bytes()
 *                       = 10 * B*S*H*D + 4 * B*H*S bytes (head-side Q, K, V,
 *                       O and dO, and the row sums); bytes beyond that,
 *                       from the next 256-byte boundary, are dS scratch as in
 *                       cpattn_attention_backward.
 * Other arguments, splits and errors as cpattn_ulysses_attention (SHAPE also
 * when B*S*H >= 2^31); causal = 1 for the causal mask.
 */
size_t cpattn_ulysses_attention_backward_workspace_bytes(int B, int H, int S, int D);
int cpattn_ulysses_attention_backward(const void *q, const void *k, const void *v,
                                      const void *out, const float *lse, const void *dout,
                                      void *dq, void *dk, void *dv, int B, int H, int S, int D,
                                      int degree, const int *seq_splits, const int *head_splits,
                                      int causal, void *workspace, size_t workspace_bytes,
                                      cpattn_stream_t stream);

/* ------------------------------------------------- no-allocation variant */

/*
 * Ulysses attention with scratch held inside the library.  The source pages
 * have no counterpart to this entry point.
 *
 * Who it is for: callers that cannot allocate device memory when they call --
 * for example a plug-in running inside another framework that owns every
 * device allocation (its caching allocator is not reachable from the plug-in),
 * or a service that reserves all GPU memory at start-up and forbids
 * cudaMalloc/cudaFree on the request path.  Such callers can still provide
 * inputs and outputs, but not the workspace cpattn_ulysses_attention needs.
 *
 * Same computation, arguments, layouts and results as cpattn_ulysses_attention
 * minus the two workspace arguments.  The four head-sharded scratch buffers
 * live in one fixed device array compiled into the library,
 * CPATTN_NOALLOC_SCRATCH_BYTES (64 MiB), present on every GPU that loads the
 * library and held until the process exits.  A problem that needs more than
 * that (8 * B*S*H*D bytes) is rejected with CPATTN_ERR_WORKSPACE before any
 * work is enqueued.
 *
 * When the memory is committed: CUDA loads the library's device code, and with
 * it this array, on a device the first time any entry point of the library
 * launches work or looks up the array there (under the default lazy module
 * loading) -- not when the shared library is loaded into the process.  A
 * caller that reserves all free GPU memory at start-up must therefore make one
 * call on each device first (for example this entry point on a small shape),
 * or that later first call fails with CPATTN_ERR_CUDA.
 *
 * The first call on a device, with that device current, looks up the array's
 * device address (cudaGetSymbolAddress) and keeps it for the life of the
 * process; make that first call on each device before any stream capture.
 * The kept address belongs to the device's primary context (the one the CUDA
 * runtime uses): do not call this entry point across a cudaDeviceReset or
 * with another context current.  Every call uses the same array, which keeps the
 * previous call's contents (nothing in it needs to start at zero): calls that
 * overlap on the GPU -- on different streams, or from different host threads
 * without ordering -- race on the array and corrupt each other's results, so
 * serialise them.  This entry point calls no cudaMalloc, cudaFree or other
 * allocating routine.
 */
#define CPATTN_NOALLOC_SCRATCH_BYTES (64u << 20)

int cpattn_ulysses_attention_noalloc(const void *q, const void *k, const void *v, void *out, float *lse,
                                     int B, int H, int S, int D, int degree, const int *seq_splits,
                                     const int *head_splits, cpattn_stream_t stream);

/* ------------------------------------------------------------- utilities */

/*
 * The uneven split used by the 'anything' workloads ([CP] "Ulysses Anything
 * Attention" removes the divisibility requirement; the page does not fix the
 * rule, this library uses front-loaded ceil): the first total % parts entries
 * get ceil(total / parts), the rest floor(total / parts).  out: host
 * int[parts].  Errors: NULL, DEGREE (parts < 1), SHAPE (total < 0).
 */
int cpattn_front_loaded_splits(int total, int parts, int *out);

/*
 * Per-rank exchange volume of one attention call, the accounting behind the
 * choice of exchange ([USP] section 5: Ulysses moves O(n*d/P) per GPU with
 * two all-to-alls, ring O(n*d) over P-1 point-to-point hops; [SP] "Choosing
 * The Attention Exchange": kv_gather moves about P/2 times the Ulysses payload
 * per rank, excluding the rank's local shard).  Host-only arithmetic on the
 * shard sizes; nothing runs on the GPU (on one GPU the exchanges are emulated
 * in memory, so these bytes are what P GPUs would send and receive).
 *
 *   mode         0 ring (K and V chunks rotate through every rank),
 *                1 Ulysses (Q, K, V to head-sharded, O back),
 *                2 kv_gather (K and V all-gathered; Q, O stay local).
 *   seq_splits   host int[degree] or NULL (equal split of S).
 *   head_splits  host int[degree] or NULL (equal split of H; Ulysses only).
 *   send, recv   host unsigned long long[degree]: bytes rank r sends/receives.
 * For rank r with S_r tokens and H_r heads, N_r = B*S_r*H*D*elem_bytes:
 *   ring, kv_gather: recv = 2 * B*(S-S_r)*H*D*e,  send = 2 * (P-1) * N_r
 *   Ulysses:        send = 3 * B*S_r*(H-H_r)*D*e + B*(S-S_r)*H_r*D*e,
 *                   recv = 3 * B*(S-S_r)*H_r*D*e + B*S_r*(H-H_r)*D*e.
 * Errors: NULL, SHAPE, DEGREE, INDIVISIBLE, SPLITS.
 */
int cpattn_exchange_bytes(int mode, int B, int H, int S, int D, int elem_bytes, int degree,
                          const int *seq_splits, const int *head_splits, unsigned long long *send,
                          unsigned long long *recv);

/*
 * Exchange-selection model: which exchange serves one attention call over P
 * ranks fastest, from the shapes and the measured speeds of the machine.
 * [SP] "Choosing The Attention Exchange": neither exchange is universally
 * faster; kv_gather moves about P/2 times the Ulysses payload but skips the
 * inverse all-to-all and keeps the local attention layout, Ulysses holds less
 * attention activation memory, and kv_gather is non-causal only.  [USP]
 * section 5: ring moves O(n*d) per GPU over P-1 sequential hops, Ulysses
 * O(n*d/P) in all-to-alls.  [SP] "Cross-Node Sequence Parallelism": the ring's
 * point-to-point K/V rotation is pipelined against attention compute.
 * Host-only arithmetic; nothing runs on the GPU.
 *
 * For every rank r the model charges (times in seconds, e = elem_bytes):
 *   ring      T = A(r, r) + sum over the P-1 later chunks c in ring order of
 *                 max(A(r, c), 2*B*S_c*H*D*e / link)
 *   ulysses   T = recv_r / link + 8*B*S_r*H*D*e / hbm + A_heads(r)
 *             (one local read+write pass over the Q, K, V and O shards)
 *   kv_gather T = recv_r / link + sum over c of A(r, c)        (no overlap)
 * where A(r, c) = 4*D*B*H*(query, key) pairs of shard r and chunk c that the
 * mask lets through / attn_flops, A_heads(r) the same for H_r heads over all
 * S tokens, recv_r the bytes of cpattn_exchange_bytes.  A mode's time is that
 * of its slowest rank.  Resident bytes: what a rank holds during attention
 *   ring      (2*S_r + 4*max_c S_c) * B*H*D*e  (Q, O, two K/V chunks in flight)
 *   ulysses   4 * B*S*H_r*D*e                  (Q, K, V, O of its heads)
 *   kv_gather (2*S_r + 2*S) * B*H*D*e          (Q, O, the full K and V)
 *
 *   env->link_gbs     interconnect bandwidth one rank receives at, GB/s (> 0)
 *   env->attn_tflops  attention throughput of one GPU, TFLOP/s (> 0)
 *   env->hbm_gbs      HBM bandwidth of one GPU, GB/s (> 0)
 *   env->causal       1: causal (kv_gather infeasible), 0: non-causal
 *   plan              written: per mode (0 ring, 1 Ulysses, 2 kv_gather) the
 *                     time (-1 if infeasible), max recv bytes, max resident
 *                     bytes and max attention FLOPs over ranks; best = the
 *                     feasible mode with the least time.
 * Ulysses is infeasible when head_splits is NULL and H % degree != 0.
 * Errors: NULL, SHAPE (a size or an env value out of range), DEGREE,
 * INDIVISIBLE (sequence), SPLITS.
 */
typedef struct {
  double link_gbs;
  double attn_tflops;
  double hbm_gbs;
  int causal;
} cpattn_exchange_env;

typedef struct {
  double seconds[3];
  unsigned long long recv_bytes[3];
  unsigned long long resident_bytes[3];
  double flops[3];
  int best;
} cpattn_exchange_plan;

int cpattn_plan_exchange(int B, int H, int S, int D, int elem_bytes, int degree,
                         const int *seq_splits, const int *head_splits,
                         const cpattn_exchange_env *env, cpattn_exchange_plan *plan);

/*
 * Synchronises `stream`, then reads and clears the device status word that the
 * kernels' bounded waits set when a pipeline wait expires.  *code receives the
 * raw word (0 = healthy; otherwise a bit per wait site; bit 6 means a kernel
 * found its shared-memory window misaligned and did nothing).  Returns CPATTN_OK,
 * CPATTN_ERR_DEVICE_TIMEOUT if the word was non-zero, or CPATTN_ERR_CUDA.
 */
int cpattn_device_status(cpattn_stream_t stream, unsigned int *code);

/*
 * Test hook for the bounded-wait mechanism: launches one block that waits on
 * an mbarrier nothing ever arrives at, with a limit of `timeout_us`
 * microseconds (1 .. 1000000), then sets the timeout bit and returns.  The
 * caller then sees CPATTN_ERR_DEVICE_TIMEOUT from cpattn_device_status.
 */
int cpattn_debug_wait_timeout(unsigned int timeout_us, cpattn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CPATTN_H */
