/*
 * gva.h — C ABI of the B200 (sm_100a) Grouped Value Attention decode library.
 *
 * Grouped Value Attention (GVA) caches only the grouped values V[T,G,d_h] and one
 * head-shared rotated positional key k_rope[T,d_r] per token.  Each query head h
 * owns a fixed map M_h (d_h x d_n) with content key K_h = V_g(h) M_h; at decode the
 * map is folded into the query, q~_h = q_h^nope M_h^T, so the score against cached
 * token j is  s_j = (q~_h . v_{j,g(h)} + RoPE(q_h^rope) . k_rope_j) * scale  and the
 * output is o_h = sum_j softmax(s)_j v_{j,g(h)}.  Content keys are never built.
 *   - onedev.kr review "GVA는 값만 캐시하고 키를 필요할 때 복원해 GQA 캐시를 절반으로
 *     줄인다", section "How it works" (어떻게 동작하나): K_h = V_g(h) M_h and the exact
 *     absorption identity q_h (v M_h)^T = (q_h M_h^T) v^T;
 *   - same review, section "What differs" (무엇과 다른가): decoupled RoPE slice d_r,
 *     k_rope = (x_j W_r) R_j^T cached separately and shared by all heads, cache
 *     N_GVA = T*G*d_h + T*d_r against N_GQA = 2*T*G*d_h;
 *   - bisque.today explainer "Grouped Value Attention matches GQA on a 47% smaller KV
 *     cache", Equation 7 (both routes give the same score, exactly).
 *
 * Conventions shared by every entry point
 *   - The caller owns every buffer.  Pointers named "device" must point to device
 *     memory of the current CUDA device; the library never allocates, frees or
 *     synchronises, and keeps no per-call state.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t passed as
 *     void*, NULL = legacy default stream).  Outputs are valid once the stream has
 *     reached that point.
 *   - Kernels are launched with programmatic dependent launch and let the next
 *     kernel on the stream start early (the combine and the first kernel of a
 *     fused step do so at entry).  A kernel of the caller's that is itself
 *     launched with programmatic stream serialization right after a call here
 *     must execute griddepcontrol.wait (cudaGridDependencySynchronize) before it
 *     reads that call's outputs; normally launched kernels need nothing.
 *   - In the other direction, the first kernel of a call reads the call's inputs
 *     (queries, key maps, new tokens, slots, positions, lengths, offsets, and the
 *     cache rows a decode attends, in a fused step those other than its new slots)
 *     before it waits for the work before it on the stream, so that the reads
 *     overlap that work's tail.  The append and absorb calls, whose outputs (cache
 *     rows, absorbed queries) the next decode reads that early, let the next
 *     kernel launch only when they have completed.
 *     A dependent may start once every thread block of the preceding kernel has
 *     exited or triggered its dependents.  Inputs from copies, from calls of this
 *     library, and from kernels that do not trigger dependents early and make their
 *     stores visible before their blocks exit (a __threadfence() at the end of
 *     the producer guarantees it) are complete by then.  A producer that triggers
 *     early must do so only after those stores are visible.
 *   - Host-side validation happens before anything is launched; a non-OK status
 *     means nothing was enqueued.  gva_last_error() returns a one-line reason for
 *     the last non-OK status of the calling thread.  GVA_ERR_CUDA reports a launch
 *     failure (cudaGetLastError after the launch).
 *   - Layouts are dense row-major.  g(h) = h / (H/G) (contiguous grouping).
 *     The query vector of a head is [content slice (d_n) | positional slice (d_r)].
 *   - RoPE on the positional slice pairs element i with i + d_r/2 and rotates the
 *     pair by pos * rope_base^(-2i/d_r); the angle is evaluated in float64.
 *   - Sequence b owns cache slots seq_offset[b] .. seq_offset[b]+seq_len[b]-1, and
 *     the token in slot seq_offset[b]+j has position j.  Sequences may be ragged.
 */
#ifndef GVA_H_
#define GVA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GVA_OK = 0,
  GVA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, inconsistent shape     */
  GVA_ERR_UNSUPPORTED = 2,   /* valid shape that no kernel here is built for    */
  GVA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required      */
  GVA_ERR_CUDA = 4           /* a CUDA runtime call or launch failed            */
} gva_status_t;

typedef enum { GVA_F32 = 0, GVA_BF16 = 1 } gva_dtype_t;

/* Flags for gva_shape_t.flags. */
#define GVA_FLAG_FMA_PATH 1u   /* decode on CUDA-core FMA instead of tensor cores  */
/* One-token GVA decode (H/G = 4, bf16 cache, d_h in {64, 128}, G in {4, 8},
 * d_r <= 32) on the tcgen05 split kernel instead of the default warp-level
 * mma.sync one.  Same result to rounding; measured slower on B200 for these thin
 * products, so it is opt-in.  Ignored for shapes it does not cover. */
#define GVA_FLAG_TCGEN05_PATH 2u

typedef struct {
  int32_t B;            /* sequences (one query token each)                       */
  int32_t H;            /* query heads                                            */
  int32_t G;            /* value groups; H % G == 0                               */
  int32_t d_h;          /* value / head width                                     */
  int32_t d_n;          /* content (unrotated) query slice width                  */
  int32_t d_r;          /* positional slice width, even, may be 0                 */
  int32_t cache_dtype;  /* gva_dtype_t of V, k_rope (and K for GQA)               */
  int32_t q_dtype;      /* gva_dtype_t of q and M                                 */
  int32_t out_dtype;    /* gva_dtype_t of the attention output                    */
  uint32_t flags;       /* GVA_FLAG_*                                             */
  double rope_base;     /* RoPE base, e.g. 10000 or 500000                        */
  float softmax_scale;  /* 0 -> 1/sqrt(d_n + d_r) (GVA) or 1/sqrt(d_h) (GQA)      */
  int32_t ctas_per_sm;  /* split-KV CTAs per SM; 0 -> library default             */
} gva_shape_t;

/* One-line description of a status code (static storage). */
const char* gva_status_string(gva_status_t status);

/* Reason for the calling thread's most recent non-OK status (thread-local). */
const char* gva_last_error(void);

/*
 * gva_absorb_query — fold each head's key map into its query and rotate the
 * positional slice (onedev.kr review, "How it works": q~_h = q_h M_h^T is computed
 * once per query token and head; "What differs": the positional slice is rotated).
 *
 *   q      device [B, H, d_n + d_r]  q_dtype
 *   M      device [H, d_h, d_n]      q_dtype   (row i of M_h maps value dim i)
 *   q_pos  device [B] int32          position of each sequence's query token
 *   q_abs  device [B, H, d_h + d_r]  float32, written:
 *            q_abs[b,h,0:d_h]      = c * (q[b,h,0:d_n] @ M[h]^T)
 *            q_abs[b,h,d_h:d_h+d_r]= c * RoPE(q[b,h,d_n:], q_pos[b])
 *          with c = softmax_scale * log2(e)  (scores come out in base-2 units).
 * Here B counts query rows, up to 262140 (e.g. B * n_query rows for
 * gva_decode_attention_multi); the decode calls take at most 4096 sequences.
 * Alignment: every pointer 16-byte aligned.  Errors: GVA_ERR_INVALID_ARG.
 */
gva_status_t gva_absorb_query(const gva_shape_t* shape, const void* q, const void* M,
                              const int32_t* q_pos, float* q_abs, void* stream);

/*
 * gva_append_cache — persist N new tokens: the grouped value is copied bit-exactly,
 * the raw positional key is rotated by its own position and rounded once (to
 * nearest, ties to even) to the cache type (onedev.kr review, "What differs":
 * k_rope = (x_j W_r) R_j^T, cached separately, d_r scalars per token).
 *
 *   v_new    device [N, G, d_h]  cache_dtype
 *   kpe_new  device [N, d_r]     cache_dtype, unrotated
 *   slot     device [N] int32    destination slot of each token
 *   pos      device [N] int32    position of each token (used by RoPE)
 *   V_cache  device [num_slots, G, d_h]  cache_dtype, updated in place
 *   kr_cache device [num_slots, d_r]     cache_dtype, updated in place
 *   err_flag device int32 or NULL: set to 1 if any slot lies outside
 *            [0, num_slots); such tokens are skipped, the others are written.
 * Two tokens with the same slot race (last writer undefined).
 * Alignment: 16 bytes for all cache/value pointers.  N == 0 is a no-op.
 */
gva_status_t gva_append_cache(const gva_shape_t* shape, int32_t N, const void* v_new,
                              const void* kpe_new, const int32_t* slot, const int32_t* pos,
                              int64_t num_slots, void* V_cache, void* kr_cache,
                              int32_t* err_flag, void* stream);

/*
 * gva_decode_workspace_size — bytes of scratch gva_decode_attention and
 * gqa_decode_attention need for `shape` on the CURRENT device (it depends on the
 * device's SM count) when the total cached tokens never exceed max_total_tokens.
 * Returns 0 for an invalid shape.
 *
 * Workspace contract: the first 4 bytes are a device status word, the next 4 a
 * work counter of the split kernel.  Zero the buffer once (e.g. cudaMemsetAsync
 * of the whole buffer) before first use; the library never clears the status
 * word, and every decode leaves the counter at 0 again.  After a decode the
 * status holds 0, or a nonzero GVA_DEVERR_* bit mask if a kernel met an
 * inconsistent input (a sequence reaching outside [0, num_slots)) or gave up a
 * bounded wait.  The rest of the buffer is overwritten every call.
 */
size_t gva_decode_workspace_size(const gva_shape_t* shape, int64_t max_total_tokens);

#define GVA_DEVERR_RANGE 1   /* some sequence's slots leave [0, num_slots); those rows read as 0 */
#define GVA_DEVERR_WAIT 2    /* a pipeline wait hit its poll or time limit; outputs invalid */

/*
 * gva_decode_attention — one GVA decode step over a (possibly ragged) batch,
 * absorbed route (onedev.kr review, "How it works": content attention reads only
 * the value cache, no key tensor; "What differs": plus the shared positional key).
 * Split-KV over all SMs with a log-sum-exp combine.
 *
 *   q_abs      device [B, H, d_h + d_r] float32 from gva_absorb_query
 *   V_cache    device [num_slots, G, d_h] cache_dtype
 *   kr_cache   device [num_slots, d_r]    cache_dtype, already rotated (ignored if d_r==0)
 *   seq_offset device [B] int32, seq_len device [B] int32 (0 allowed)
 *   max_total_tokens  upper bound of sum(seq_len) (host value, sizes the split)
 *   out        device [B, H, d_h] out_dtype   o_h = sum_j p_j v_{j,g(h)}
 *   lse        device [B, H] float32 or NULL: natural-log log-sum-exp of the scaled
 *              scores (-inf for an empty sequence, whose output is 0)
 *   workspace  device, ws_bytes >= gva_decode_workspace_size(shape, max_total_tokens)
 * Alignment: 16 bytes for all pointers; V_cache rows (G*d_h*elt) and k_rope rows
 * (d_r*elt) must be multiples of 16 bytes.  Concurrent calls on different streams
 * must use different workspaces.
 */
gva_status_t gva_decode_attention(const gva_shape_t* shape, const float* q_abs,
                                  const void* V_cache, const void* kr_cache,
                                  const int32_t* seq_offset, const int32_t* seq_len,
                                  int64_t max_total_tokens, int64_t num_slots, void* out,
                                  float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * gqa_decode_attention — same-shape grouped-query attention decode, the matched
 * baseline of every page (it caches a key AND a value per group and token,
 * N_GQA = 2*T*G*d_h).  Same split and combine as gva_decode_attention.
 *
 *   q          device [B, H, d_h] q_dtype, already rotated
 *   K_cache, V_cache  device [num_slots, G, d_h] cache_dtype (keys already rotated)
 *   scale      shape->softmax_scale, 0 -> 1/sqrt(d_h); shape->d_n and d_r are ignored
 * Other arguments, alignment and workspace as for gva_decode_attention.
 */
gva_status_t gqa_decode_attention(const gva_shape_t* shape, const void* q, const void* K_cache,
                                  const void* V_cache, const int32_t* seq_offset,
                                  const int32_t* seq_len, int64_t max_total_tokens,
                                  int64_t num_slots, void* out, float* lse, void* workspace,
                                  size_t ws_bytes, void* stream);

/*
 * gqa_append_cache — persist N new tokens into the same-shape GQA cache, the
 * matched baseline that keeps a key AND a value per group and token (onedev.kr
 * review, "What differs": N_GQA = 2*T*G*d_h).  The value is copied bit-exactly;
 * each group's key is rotated by the token's position over the whole head width
 * (pair i with i + d_h/2, angle pos * rope_base^(-2i/d_h) in float64) and stored
 * rounded once (to nearest, ties to even) to the cache type.
 *
 *   k_new, v_new      device [N, G, d_h] cache_dtype (k_new unrotated)
 *   slot, pos         device [N] int32: destination slot and position of each token
 *   K_cache, V_cache  device [num_slots, G, d_h] cache_dtype, updated in place
 *   err_flag          device int32 or NULL: set to 1 if a slot lies outside
 *                     [0, num_slots); such tokens are skipped, the others written
 * Shape: d_n and d_r are ignored; d_h even and <= 128; rope_base > 0.
 * Alignment: 16 bytes for every pointer; G*d_h*elt a multiple of 16 bytes.
 * Errors: GVA_ERR_INVALID_ARG, GVA_ERR_UNSUPPORTED (odd or too wide d_h).
 * N == 0 is a no-op.  Two tokens with the same slot race.
 */
gva_status_t gqa_append_cache(const gva_shape_t* shape, int32_t N, const void* k_new,
                              const void* v_new, const int32_t* slot, const int32_t* pos,
                              int64_t num_slots, void* K_cache, void* V_cache, int32_t* err_flag,
                              void* stream);

/*
 * gqa_decode_step — one full decode step of the same-shape GQA baseline, the
 * counterpart of gva_decode_step used to compare whole steps: the query of every
 * sequence is rotated over d_h at q_pos[b] into q_rot (float32, unscaled), the
 * n_new new tokens are appended as by gqa_append_cache, then gqa_decode_attention
 * runs on q_rot (onedev.kr review, "What differs": GQA caches and reads a key and
 * a value per group and token).  One kernel does the rotation and the append; the
 * decode is launched behind it and streams every cache tile that holds no new
 * slot before that kernel finishes.
 *
 *   q       device [B, H, d_h] q_dtype, unrotated;  q_pos device [B] int32
 *   q_rot   device [B, H, d_h] float32, written (the rotated query)
 *   k_new, v_new, slot, pos, K_cache, V_cache, num_slots, err_flag: as gqa_append_cache
 *   seq_offset, seq_len, max_total_tokens, out, lse, workspace: as
 *           gqa_decode_attention (seq_len already counts the new tokens; the
 *           workspace size is gva_decode_workspace_size of the shape)
 * Errors as gqa_append_cache and gqa_decode_attention; all validation happens
 * before the first launch.
 */
gva_status_t gqa_decode_step(const gva_shape_t* shape, const void* q, const int32_t* q_pos,
                             int32_t n_new, const void* k_new, const void* v_new,
                             const int32_t* slot, const int32_t* pos, void* K_cache,
                             void* V_cache, int64_t num_slots, const int32_t* seq_offset,
                             const int32_t* seq_len, int64_t max_total_tokens, float* q_rot,
                             void* out, float* lse, int32_t* err_flag, void* workspace,
                             size_t ws_bytes, void* stream);

/*
 * gva_decode_step — one full GVA decode step: gva_append_cache of the n_new new
 * tokens, gva_absorb_query, then gva_decode_attention, enqueued on `stream` in
 * that order (onedev.kr review, "How it works" and "What differs": the new
 * token's value and rotated positional key are cached, the query is absorbed,
 * content attention reads only the value cache).  Arguments are those of the
 * three calls; seq_len must already count the new tokens, q_abs is the caller's
 * [B, H, d_h + d_r] float32 buffer for the absorbed queries, err_flag may be NULL.
 * Because the append finishes before the decode is launched, the decode starts
 * streaming the cache while the absorb kernel still runs.  Validation of all three
 * parts happens before the first launch, except for errors only the append or
 * absorb checks catch, in which case the earlier parts may have been enqueued.
 */
gva_status_t gva_decode_step(const gva_shape_t* shape, const void* q, const void* M,
                             const int32_t* q_pos, int32_t n_new, const void* v_new,
                             const void* kpe_new, const int32_t* slot, const int32_t* pos,
                             void* V_cache, void* kr_cache, int64_t num_slots,
                             const int32_t* seq_offset, const int32_t* seq_len,
                             int64_t max_total_tokens, float* q_abs, void* out, float* lse,
                             int32_t* err_flag, void* workspace, size_t ws_bytes, void* stream);

/*
 * gva_decode_attention_multi — decode of n_query new tokens per sequence at once
 * (e.g. verifying draft tokens in speculative decoding), causal among them: the
 * new tokens are already appended and occupy positions L-n_query .. L-1 of each
 * sequence (L = seq_len[b]); query i attends cache positions 0 .. L-n_query+i.
 * Same absorbed route as gva_decode_attention (onedev.kr review, "How it works"
 * and "What differs"); each cache tile is read once for all queries and heads of
 * its group.
 *
 *   q_abs  device [B, n_query, H, d_h + d_r] float32: gva_absorb_query run on the
 *          B*n_query query tokens (shape->B = B*n_query, q_pos = their positions)
 *   out    device [B, n_query, H, d_h] out_dtype; lse device [B, n_query, H] or NULL
 *   workspace: gva_decode_workspace_size_multi(shape, n_query, max_total_tokens)
 *   Other arguments as gva_decode_attention.  n_query = 1 is gva_decode_attention.
 *
 * Two kernels, by the number of query columns per value group, (H/G)*n_query:
 *  - up to 8 (speculative blocks): the split-KV decode kernel (mma.sync), the
 *    columns sharing each tile, then the combine; bf16 cache, d_h in {64, 128};
 *  - more than 8 (chunked prefill, long drafts): the tcgen05 kernel, one CTA per
 *    128 query rows (token x head) of a group, scores and outputs accumulated in
 *    tensor memory, output written directly (the workspace only carries the
 *    status word); bf16 cache, d_h in {64, 128}, d_r a multiple of 8 up to 32,
 *    H/G dividing 128.
 * Other shapes return GVA_ERR_UNSUPPORTED.
 */
size_t gva_decode_workspace_size_multi(const gva_shape_t* shape, int32_t n_query,
                                       int64_t max_total_tokens);

gva_status_t gva_decode_attention_multi(const gva_shape_t* shape, int32_t n_query,
                                        const float* q_abs, const void* V_cache,
                                        const void* kr_cache, const int32_t* seq_offset,
                                        const int32_t* seq_len, int64_t max_total_tokens,
                                        int64_t num_slots, void* out, float* lse,
                                        void* workspace, size_t ws_bytes, void* stream);

/*
 * gva_shared_kv_decode_attention — decode with shared keys and values (K = V):
 * the special case of GVA with M_h = I and no positional slice, the first design
 * the authors tried, whose cache is exactly half of the matched GQA cache
 * (onedev.kr review, "How it is used" (어떻게 쓰나)).  Scores s_j = q_h . v_{j,g(h)} / sqrt(d_h),
 * softmax over the L_b cached rows, o_h = sum_j p_j v_{j,g(h)}.  No absorb step:
 * the raw query is read in q_dtype and scaled inside the decode kernel.
 *
 *   shape      d_r == 0 and d_n == d_h (else GVA_ERR_INVALID_ARG); softmax_scale 0
 *              -> 1/sqrt(d_h)
 *   q          device [B, H, d_h] q_dtype (RoPE, if the model uses it, already applied)
 *   V_cache    device [num_slots, G, d_h] cache_dtype: keys and values
 *   other arguments, workspace (gva_decode_workspace_size of the same shape),
 *   alignment and errors as for gva_decode_attention.
 */
gva_status_t gva_shared_kv_decode_attention(const gva_shape_t* shape, const void* q,
                                            const void* V_cache, const int32_t* seq_offset,
                                            const int32_t* seq_len, int64_t max_total_tokens,
                                            int64_t num_slots, void* out, float* lse,
                                            void* workspace, size_t ws_bytes, void* stream);

/*
 * gva_merge_states — merge R attention states of the same queries computed over
 * disjoint parts of each sequence's cache, e.g. one part per GPU when one long
 * sequence's cache is split across GPUs.  The pages have no counterpart (they
 * run no long-context or multi-GPU test: onedev.kr review, "Premises and
 * limits"); the merge is the exact decomposition of softmax attention:
 *   lse = log sum_r exp(lse_r),   out = sum_r exp(lse_r - lse) * out_r.
 *
 *   outs  device [R, B, H, d_h] float32  normalised outputs of the R parts
 *   lses  device [R, B, H]      float32  their natural-log lse (-inf: empty part,
 *                                        whose output is ignored)
 *   out   device [B, H, d_h] out_dtype; lse device [B, H] float32 or NULL
 *   Only shape->B, H, d_h and out_dtype are used.  All-empty -> 0 and -inf.
 */
gva_status_t gva_merge_states(const gva_shape_t* shape, int32_t R, const float* outs,
                              const float* lses, void* out, float* lse, void* stream);

/*
 * gva_decode_attention_noalloc — gva_decode_attention for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is an interface
 * convenience of this library.
 *
 * Some callers have no way to obtain scratch memory: code that runs while a
 * stream is being captured into a CUDA graph (cudaMalloc is not allowed there),
 * plug-ins that only receive input and output buffers from a host framework whose
 * caching allocator owns all other device memory, and latency-critical paths that
 * must not call cudaMalloc because it can synchronise the device.  This entry
 * point needs no workspace: the split-KV scratch is a fixed array of
 * GVA_NOALLOC_SCRATCH_BYTES in this library's own device memory, which every GPU
 * that loads the library holds until the process exits.  It allocates nothing
 * (no cudaMalloc, cudaFree or allocating library routine); the caller still
 * passes every input and output, as for gva_decode_attention.
 *
 *   Arguments, layouts, alignment and results: as gva_decode_attention.
 *   Errors: GVA_ERR_WORKSPACE if the shape needs more scratch than
 *   GVA_NOALLOC_SCRATCH_BYTES (gva_decode_workspace_size tells); GVA_ERR_CUDA if
 *   the scratch's device address cannot be found.
 *   The first call on each device looks up the scratch's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before
 *   any stream capture.  Every accepted call zeroes the scratch's status word on
 *   `stream` before its kernels run; a call rejected on the host enqueues nothing
 *   and leaves the scratch untouched.  The call's device errors (GVA_DEVERR_*) stay
 *   in that word until the next call: read them with gva_noalloc_status.
 *   All calls on a device share the one scratch array, which keeps the last call's
 *   contents: calls whose executions overlap on the GPU (different streams, or
 *   concurrent graphs) race and give wrong results.  Serialise them.
 */
#define GVA_NOALLOC_SCRATCH_BYTES (8u << 20)

gva_status_t gva_decode_attention_noalloc(const gva_shape_t* shape, const float* q_abs,
                                          const void* V_cache, const void* kr_cache,
                                          const int32_t* seq_offset, const int32_t* seq_len,
                                          int64_t max_total_tokens, int64_t num_slots, void* out,
                                          float* lse, void* stream);

/*
 * gva_noalloc_status — the device status word of the most recent
 * gva_decode_attention_noalloc call on the current device, i.e. the first 4 bytes
 * of its static scratch: 0, or a GVA_DEVERR_* bit mask (GVA_DEVERR_RANGE: a
 * sequence reached outside [0, num_slots) and its missing rows read as 0;
 * GVA_DEVERR_WAIT: a bounded pipeline wait gave up and the outputs are invalid).
 * The paper has no counterpart: an interface convenience of this library for
 * callers without a workspace of their own.
 *
 *   status_out  device memory or page-locked host memory, one int32: receives
 *               the word by an asynchronous copy enqueued on `stream`; it is valid
 *               once the stream reaches that point (e.g. after
 *               cudaStreamSynchronize).  Enqueue it behind the decode it checks,
 *               on the same stream, and before the next no-allocation decode.
 * Allocates nothing.  Errors: GVA_ERR_INVALID_ARG (NULL status_out), GVA_ERR_CUDA
 * (the scratch's address or the copy failed).
 */
gva_status_t gva_noalloc_status(int32_t* status_out, void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* GVA_H_ */
