/*
 * lsh_attn.h -- C ABI of liblsh_attn.so, the B200 (sm_100a) LSH attention
 * forward pass: shared-QK attention restricted by random-rotation hashing,
 * as described in "Reformer: The Efficient Transformer" (arXiv 2001.04451v2):
 *   section 2 "LSH attention"     -- hash h(x) = argmax([xR; -xR]), sort by
 *                                    bucket, attend within sorted chunks;
 *   section 2 "Causal masking"    -- positions follow the same permutation,
 *                                    future positions are masked, a token may
 *                                    attend to itself only when nothing else
 *                                    is available;
 *   section 5 "Shared query-key space" -- one projection serves as query and
 *                                    key; keys are normalised;
 *   Appendix A "Multi-round attention" / "Implementation" / "Masking" --
 *                                    n_hashes independent rounds, each giving
 *                                    its own output, combined afterwards.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor arguments are DEVICE pointers (cudaMalloc'd or equivalent)
 *    unless the name ends in _host.  The caller owns every buffer, including
 *    the workspace, and the library keeps no pointer after a call returns.
 *    The library allocates nothing: the stage calls and the fused call take
 *    their temporary memory from caller workspaces (sized by the
 *    *_workspace_size queries).  The two places where it holds device
 *    resources of its own are stated at their calls: lsh_attn_forward_host's
 *    streams and events, and lsh_attn_forward_noalloc's built-in scratch.
 *  - Every device pointer must be 16-byte aligned.  Tensors are dense,
 *    row-major, last dimension fastest.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  All work is enqueued on it; no call synchronises the host
 *    except lsh_attn_device_check().
 *  - Arguments are checked on the host before anything is launched.  A call
 *    that returns anything but LSH_OK has launched nothing, except
 *    LSH_ERR_CUDA (a launch or copy failed part-way; lsh_attn_last_error()
 *    has the CUDA message).
 *  - Shapes (see lsh_shape): B batch, H heads, L seq_len, d d_k,
 *    n_h n_hashes, n_b n_buckets, c chunk_len.
 *  - Besides those resources, the library keeps no state between calls
 *    except one device word that records a kernel's bounded wait running out
 *    (see lsh_attn_device_check).
 */
#ifndef LSH_ATTN_H_
#define LSH_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LSH_ATTN_VERSION 1

#if defined(__GNUC__)
#define LSH_ATTN_API __attribute__((visibility("default")))
#else
#define LSH_ATTN_API
#endif

typedef enum lsh_status {
  LSH_OK = 0,
  LSH_ERR_INVALID_ARG = 1,     /* null/misaligned pointer, bad size or flag */
  LSH_ERR_UNSUPPORTED = 2,     /* valid request this library cannot serve  */
  LSH_ERR_WORKSPACE = 3,       /* workspace or staging buffer too small     */
  LSH_ERR_CUDA = 4,            /* a CUDA launch or copy failed              */
  LSH_ERR_DEVICE_TIMEOUT = 5   /* a kernel's bounded wait ran out           */
} lsh_status;

typedef enum lsh_dtype {
  LSH_F32 = 0,                 /* float32 qk, v, rotations, out, o_rounds   */
  LSH_BF16 = 1                 /* bfloat16 qk, v, rotations, out, o_rounds  */
} lsh_dtype;

/* lsh_shape.flags bits */
#define LSH_FLAG_PORTABLE 1u   /* use the CUDA-core kernels even where the
                                  tensor-core (tcgen05) kernels apply; for
                                  cross-checking the two kernel families   */
#define LSH_FLAG_DEDUP 2u      /* duplicate-count correction ("Reformer: The
                                  Efficient Transformer", Appendix A "Multi-
                                  round LSH attention", its "Duplicate
                                  handling" item): a key that falls in a
                                  query's window in N rounds has log N
                                  subtracted from its score in each of them,
                                  so the combined output weighs every
                                  distinct key once.  N counts the rounds r
                                  with chunk(undo_r[i]) - chunk(undo_r[j]) in
                                  {0, 1}.  Runs on the tensor-core attention
                                  for n_h <= 8 where it has a plan for the
                                  (c, d) pair, else on the CUDA-core kernel;
                                  the stage call is lsh_attn_chunked_fwd_ex. */
#define LSH_FLAG_BUCKET_MASK 4u /* bucket-equality mask (section 2 "LSH
                                  attention": a query attends only to
                                  targets in its own hash bucket): inside a
                                  window, keys whose bucket in that round
                                  differs from the query's are not attended.
                                  Runs on the tensor-core attention (on the
                                  CUDA-core kernel together with
                                  LSH_FLAG_DEDUP); the stage call is
                                  lsh_attn_chunked_fwd_ex.                 */
#define LSH_FLAG_KMEANS 8u     /* routing-style bucket assignment (the pages
                                  name online k-means for the Routing
                                  Transformer): `rotations` holds centroids
                                  [n_h, d, n_b], one set per round, and a
                                  token goes to the bucket of the centroid
                                  with the largest dot product (lowest index
                                  on ties); n_b may then be any value in
                                  [2, 32768].  bf16 with d in {64, 128} and
                                  n_b a multiple of 32 runs on the tensor-
                                  core hash kernel, other shapes on the
                                  CUDA-core one.                            */

typedef struct lsh_shape {
  int32_t batch;       /* B >= 1                                             */
  int32_t heads;       /* H >= 1                                             */
  int32_t seq_len;     /* L >= 1, < 2^31 / n_h                                */
  int32_t d_k;         /* d: 8..256, a multiple of 8                         */
  int32_t n_hashes;    /* n_h >= 1 hashing rounds                            */
  int32_t n_buckets;   /* n_b: 1, or even with 2 <= n_b <= 32768; any value
                          in [2, 32768] with LSH_FLAG_KMEANS                 */
  int32_t chunk_len;   /* c >= 1; when c does not divide L the last chunk of
                          the sorted order holds the L mod c remaining slots */
  int32_t causal;      /* 0 or 1                                             */
  int32_t dtype;       /* lsh_dtype of the floating-point tensors            */
  uint32_t flags;      /* LSH_FLAG_* bits, 0 by default                      */
} lsh_shape;

/* ---------------------------------------------------------------------- *
 * Stage 1: hash.  Section 2 "LSH attention": h(x) = argmax([xR; -xR]) with
 * a random projection R per round (Appendix A).
 *   qk        [B, H, L, d]        dtype, the shared query/key vectors.
 *   rotations [n_h, d, n_b/2]     dtype, one R per round, shared by all
 *                                 (b, h); must be NULL when n_b == 1 (every
 *                                 token then lands in bucket 0).
 *   buckets   [B, H, n_h, L]      int16 out: the argmax index in [0, n_b);
 *                                 ties go to the lowest index of [xR; -xR].
 *                                 Projections are accumulated in float32
 *                                 (exact bf16 products), so a position whose
 *                                 top two entries of [xR; -xR] are within
 *                                 float32 rounding may differ from an exact
 *                                 evaluation.
 *   inv_norm  [B, H, L]           float32 out: 1 / ||qk_i||_2, 0 for a zero row
 *                                 (the key normalisation of section 5).
 * ---------------------------------------------------------------------- */
LSH_ATTN_API lsh_status lsh_attn_hash(const lsh_shape* shape, const void* qk, const void* rotations,
                         int16_t* buckets, float* inv_norm, void* stream);

/* ---------------------------------------------------------------------- *
 * Stage 2: sort.  Section 2 / Appendix A "Implementation": per (b, h, round)
 * the positions ordered by bucket, positions increasing inside a bucket
 * (a stable sort by bucket, i.e. by the key (round, bucket, position)).
 *   buckets [B, H, n_h, L]  int16 in, values in [0, n_b).
 *   perm    [B, H, n_h, L]  int32 out: perm[.., s] = position at sorted slot s.
 *   undo    [B, H, n_h, L]  int32 out, may be NULL: undo[.., perm[.., s]] = s.
 *   counts  [B, H, n_h, n_b] int32 out, may be NULL: tokens per bucket.
 *   workspace  device memory of at least lsh_attn_sort_workspace_size()
 *              bytes (n_h * B * H * ceil(L / 2048) * n_b * 4: the per-tile
 *              bucket counts); 16-byte aligned; contents on entry ignored.
 * Bucket ids outside [0, n_b) are undefined behaviour (stage 1 never makes
 * them); the kernels do not read or write out of bounds for them.
 * A workspace smaller than the query's answer returns LSH_ERR_WORKSPACE.
 * The per-bucket counts come out of this stage, not out of stage 1: the
 * sort counts every tile of keys anyway (its first kernel), so the hash
 * needs no histogram of its own.
 * ---------------------------------------------------------------------- */
LSH_ATTN_API lsh_status lsh_attn_sort_workspace_size(const lsh_shape* shape, size_t* bytes);
LSH_ATTN_API lsh_status lsh_attn_sort(const lsh_shape* shape, const int16_t* buckets, int32_t* perm,
                         int32_t* undo, int32_t* counts, void* workspace,
                         size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------- *
 * Stage 3: chunked attention of every round, results stored at ORIGINAL
 * positions (the unsort is folded into the store).  Section 2 "LSH
 * attention" / "Causal masking"; section 5 "Shared query-key space";
 * Appendix A "Implementation" / "Masking".  For round r, sorted slot s sits
 * in chunk k = s / c; its window is chunk k-1 (if k > 0) and chunk k.  The
 * score of query i and key j is (qk_i . qk_j) * inv_norm_j / sqrt(d); the
 * score of j == i is replaced by -1e5; with causal, j > i is excluded.
 *   qk, v       [B, H, L, d]      dtype.
 *   inv_norm    [B, H, L]         float32 (from stage 1).
 *   perm        [B, H, n_h, L]    int32 (from stage 2).
 *   o_rounds    [B, H, n_h, L, d] dtype out: softmax-weighted v per round.
 *               16-byte alignment suffices; with 32-byte alignment (every
 *               cudaMalloc'd buffer) the bf16 kernels write it in 32-byte
 *               stores, which is faster.
 *   lse_rounds  [B, H, n_h, L]    float32 out: log-sum-exp of the scores.
 * ---------------------------------------------------------------------- */
LSH_ATTN_API lsh_status lsh_attn_chunked_fwd(const lsh_shape* shape, const void* qk, const void* v,
                                const float* inv_norm, const int32_t* perm, void* o_rounds,
                                float* lse_rounds, void* stream);

/* ---------------------------------------------------------------------- *
 * Stage 3 for the variants (LSH_FLAG_DEDUP, LSH_FLAG_BUCKET_MASK, set in
 * shape->flags): as lsh_attn_chunked_fwd, plus
 *   undo    [B, H, n_h, L] int32 in, required with LSH_FLAG_DEDUP: every
 *           round's inverse permutation (the undo output of lsh_attn_sort),
 *           from which the kernel counts, for each (query, key) pair, the
 *           rounds whose window holds the pair; else may be NULL.
 *   buckets [B, H, n_h, L] int16 in, required with LSH_FLAG_BUCKET_MASK:
 *           the bucket ids of stage 1; else may be NULL.
 * ---------------------------------------------------------------------- */
LSH_ATTN_API lsh_status lsh_attn_chunked_fwd_ex(const lsh_shape* shape, const void* qk,
                                   const void* v, const float* inv_norm,
                                   const int32_t* perm, const int32_t* undo,
                                   const int16_t* buckets, void* o_rounds,
                                   float* lse_rounds, void* stream);

/* ---------------------------------------------------------------------- *
 * Stage 4: combine.  Appendix A "Multi-round attention": each round's output
 * is combined with weight exp(lse_r - LSE), LSE = logsumexp over rounds.
 *   o_rounds [B, H, n_h, L, d] dtype; lse_rounds [B, H, n_h, L] float32.
 *   out      [B, H, L, d] dtype out; lse [B, H, L] float32 out (= LSE).
 * ---------------------------------------------------------------------- */
LSH_ATTN_API lsh_status lsh_attn_combine(const lsh_shape* shape, const void* o_rounds,
                            const float* lse_rounds, void* out, float* lse, void* stream);

/* ---------------------------------------------------------------------- *
 * The whole forward pass (stages 1-4) on one stream, no host sync.
 * Produces the same out/lse as the four stage calls in sequence.
 *   workspace: device scratch of at least lsh_attn_forward_workspace_size()
 *   bytes, 256-byte aligned; its contents on entry do not matter and on
 *   return are unspecified.  Two calls in flight at once need two workspaces.
 * ---------------------------------------------------------------------- */
LSH_ATTN_API lsh_status lsh_attn_forward_workspace_size(const lsh_shape* shape, size_t* bytes);

LSH_ATTN_API lsh_status lsh_attn_forward(const lsh_shape* shape, const void* qk, const void* v,
                            const void* rotations, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------- *
 * Backward of the forward pass with the buckets and their sort held fixed
 * (the hash is piecewise constant: no gradient flows through bucket ids).
 * Gradients of `out` w.r.t. the shared qk and v for an upstream gradient
 * dout, from the multiset form of the combined output (section 2 "LSH
 * attention", Appendix A): with LSE the forward's lse output,
 *   dv_j  += exp(s_ij - LSE_i) dout_i                 over every window pair,
 *   ds_ij  = exp(s_ij - LSE_i) (dout_i . v_j - dout_i . out_i),
 * into the query and the normalised key (the self pair's -1e5 is a constant).
 *   qk, v, out, dout [B, H, L, d] dtype in; inv_norm [B, H, L] float32 and
 *   perm [B, H, n_h, L] int32 from stages 1-2; lse [B, H, L] float32 from
 *   the combine; dqk, dv [B, H, L, d] float32 out.
 *   workspace: at least lsh_attn_backward_workspace_size() bytes, 256-byte
 *   aligned.  CUDA cores with float32 atomics (the summation order, and so
 *   the last bits, can differ between runs).  The variant flags are not
 *   supported here (LSH_ERR_UNSUPPORTED).
 * ---------------------------------------------------------------------- */
LSH_ATTN_API lsh_status lsh_attn_backward_workspace_size(const lsh_shape* shape, size_t* bytes);

LSH_ATTN_API lsh_status lsh_attn_backward(const lsh_shape* shape, const void* qk, const void* v,
                             const float* inv_norm, const int32_t* perm, const void* out,
                             const float* lse, const void* dout, float* dqk, float* dv,
                             void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------- *
 * The forward pass from HOST buffers: copies qk, v and rotations to the
 * device, runs the forward pass, and copies out and lse back.  The (batch,
 * head) pairs are independent, so they go in up to 8 groups through three
 * library-owned streams (copy in, compute, copy out): a group's inputs cross
 * PCIe while the previous group computes and the one before it copies back;
 * a group's qk crosses before its v, and its hash and sort start on qk alone.
 * The work starts after what is already queued on `stream`, and `stream`
 * waits for all of it, so the caller synchronises `stream` before reading
 * out_host / lse_host.  Calls on one device enqueue one at a time (a mutex
 * guards the shared streams).  Host buffers should be page-locked for the
 * copies to overlap.  On an error after the first copy was queued, `stream`
 * still waits for everything already queued (which reads and writes the
 * caller's buffers), so synchronise it before freeing them; out_host and
 * lse_host are then undefined.
 *   device_buffer: caller-owned device memory of at least
 *   lsh_attn_forward_host_device_bytes() bytes, 256-byte aligned; it holds the
 *   device copies of the inputs and outputs plus the workspace.
 * ---------------------------------------------------------------------- */
LSH_ATTN_API lsh_status lsh_attn_forward_host_device_bytes(const lsh_shape* shape, size_t* bytes);

LSH_ATTN_API lsh_status lsh_attn_forward_host(const lsh_shape* shape, const void* qk_host,
                                 const void* v_host, const void* rotations_host,
                                 void* out_host, float* lse_host, void* device_buffer,
                                 size_t device_bytes, void* stream);

/* ---------------------------------------------------------------------- *
 * The forward pass without any device allocation or caller workspace.
 * (The paper has no counterpart: this is a deployment aid of this library.)
 *
 * For callers that cannot allocate device memory: a plugin inside a host
 * framework that owns all device memory through its own pool and hands the
 * plugin only its input and output buffers, or a latency-critical path that
 * must not call cudaMalloc because it can synchronise the whole device and
 * take an unpredictable time.  Same arguments and results as
 * lsh_attn_forward, minus the workspace: the intermediates live in a scratch
 * array of LSH_ATTN_NOALLOC_SCRATCH_BYTES built into the library.
 *  - The scratch occupies that much device memory on every GPU whose
 *    context has loaded the library's device code, until the process exits.
 *    Under lazy module loading (CUDA's default, CUDA_MODULE_LOADING=LAZY)
 *    that is the GPUs where this call has run, from its first call there;
 *    with CUDA_MODULE_LOADING=EAGER it is every GPU on which the process
 *    creates a context once the library is loaded.
 *  - The first successful call on a device resolves the scratch's device
 *    address (cudaGetSymbolAddress) with that device current and keeps it;
 *    a failed lookup is retried on the next call.  Make that first call
 *    before any stream capture.
 *  - Problems whose workspace (lsh_attn_forward_workspace_size) exceeds
 *    LSH_ATTN_NOALLOC_SCRATCH_BYTES are rejected with LSH_ERR_WORKSPACE
 *    before anything is launched.
 *  - Every call on a device shares the one scratch and leaves its contents
 *    behind; nothing in it needs to start at zero.  Calls that overlap on
 *    the GPU (different streams, or different host threads, without ordering
 *    between them) race on the scratch and give wrong results: order them.
 *  - Calls no cudaMalloc, cudaFree or any other allocating routine.
 * ---------------------------------------------------------------------- */
#define LSH_ATTN_NOALLOC_SCRATCH_BYTES (64u << 20)

LSH_ATTN_API lsh_status lsh_attn_forward_noalloc(const lsh_shape* shape, const void* qk,
                                                 const void* v, const void* rotations,
                                                 void* out, float* lse, void* stream);

/* ---------------------------------------------------------------------- *
 * Diagnostics.
 *   lsh_attn_status_string: static text for a status.
 *   lsh_attn_last_error: detail of the last failing call on this host
 *   thread (static storage, overwritten by the next failure).
 *   lsh_attn_device_check: synchronises `stream`, then reads and clears the
 *   device word that a kernel sets when one of its bounded waits runs out;
 *   returns LSH_ERR_DEVICE_TIMEOUT if it was set, LSH_ERR_CUDA if the
 *   synchronisation failed, LSH_OK otherwise.
 *   lsh_attn_version: LSH_ATTN_VERSION of the built library.
 * ---------------------------------------------------------------------- */
LSH_ATTN_API const char* lsh_attn_status_string(lsh_status status);
LSH_ATTN_API const char* lsh_attn_last_error(void);
LSH_ATTN_API lsh_status lsh_attn_device_check(void* stream);
LSH_ATTN_API int lsh_attn_version(void);

/* Number of CUDA kernels this library has launched in this process so far
 * (every stage, variant and entry point; host-side count taken at launch).
 * A diagnostic for benchmarks that report how many of their kernels ran in a
 * timed region: read it before and after.  Thread-safe; never reset. */
LSH_ATTN_API unsigned long long lsh_attn_kernel_launches(void);

/* Test hook for the failure-detection path.  Every wait inside this
 * library's tensor-core kernels is bounded (2 s); when one runs out the
 * kernel records an error word, every role of the CTA leaves its loop, work
 * already in flight is drained and the kernel returns, and
 * lsh_attn_device_check reports LSH_ERR_DEVICE_TIMEOUT.  This call sets the
 * limit, in ns, of the first wait of the tensor-core hash's MMA thread (for
 * the input tile of every CTA) for the hash launches that follow: 0 makes
 * that wait give up at once, so a test can exercise the path without any
 * fault or hang.  Returns the previous limit; pass it back to restore the
 * normal behaviour.  Process-wide; not for use while other threads launch. */
LSH_ATTN_API unsigned long long lsh_attn_test_hash_first_wait(unsigned long long ns);

#ifdef __cplusplus
}
#endif

#endif /* LSH_ATTN_H_ */
