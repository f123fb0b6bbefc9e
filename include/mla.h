/*
 * mla.h -- C ABI of libmla: multi-head latent attention computed on a paged,
 * compressed latent cache, with weight absorption and decoupled RoPE, for
 * NVIDIA B200 (sm_100a).
 *
 * The method (pages named by title and section):
 *   - "ai-decoupled-rope-mla" (operatorworld), decoupled-RoPE section: each
 *     token caches a latent c_t = W_DKV h_t and a small position key
 *     k_R,t = RoPE_t(W_KR h_t); the query has a content part q_C and a rotated
 *     position part q_R; the score adds a content term and a position term.
 *   - "Latent Attention Meets RoPE" (sahipadhai), "Two small, telling details":
 *     the position key is one vector shared by all heads, and only the latent
 *     and that key are cached.
 *   - "ai-decoupled-rope-mla", absorption equations: q~ = W_UK^T q_C scores the
 *     latent directly, and the output is W_UV applied to sum_t alpha_t c_t.
 *   - "Detailed Illustration of the Problem" (notion), Step 1: an optional
 *     query latent c_Q = W_DQ h feeds the query projections.
 *
 * Conventions for every call:
 *   - All tensor arguments are DEVICE pointers owned by the caller, dense,
 *     row-major, with the element type given by mla_dims.dtype (fp32 or
 *     bf16) unless stated otherwise.  Index arrays are int32.
 *   - Every call is asynchronous on `stream`.  Argument errors are reported
 *     before anything is launched.  Errors found on the device (a page id out
 *     of range, a length out of range) are OR-ed into an error word at the
 *     start of the caller's workspace and never trap; mla_get_error reads it.
 *   - The library calls no device-memory allocator.  Scratch space is the
 *     caller's `workspace`, sized by the *_workspace_bytes queries; the
 *     workspace of a call must not be used by another call that may run at
 *     the same time.  (The workspace-free append keeps a fixed ~2 MiB array in
 *     the library's own device memory instead, see below.)  Decode creates,
 *     on its first call in a host thread on a device, one non-blocking CUDA
 *     stream and two events of its own: the attention schedule runs there
 *     beside the query projections, forked from and joined back into
 *     `stream` (which a CUDA graph capture of `stream` records as ordinary
 *     dependencies); make that first call before any stream capture.
 *   - Cache layout: [num_pages, page_size, d_cr]; row (page p, slot s) holds
 *     [c_t (d_c) | k_R,t (d_r)] (d_cr = d_c + d_r; with per-head RoPE keys
 *     d_cr = d_c + n_h*d_r, see mla_dims) for the token whose position is
 *     j*page_size + s, where page_table[seq*max_pages + j] == p.
 *   - Weight orientation is column-vector, y = W x: W_DKV [d_c, d_model],
 *     W_KR [d_r, d_model], W_DQ [d_cq, d_model], W_UQ [n_h*d_h, d_in],
 *     W_QR [n_h*d_r, d_in], W_UK [n_h*d_h, d_c], W_UV [n_h*d_v, d_c], where
 *     d_in = d_cq when d_cq > 0, else d_model.  Rows h*d_h .. h*d_h+d_h-1 of
 *     W_UK (and likewise W_UQ, W_QR, W_UV) belong to head h.
 *   - RoPE rotates interleaved pairs (2i, 2i+1) by pos * rope_base^(-2i/d_r);
 *     the pages print only the rotation family, so the frequencies and the
 *     pairing are the reading this library takes.
 *   - A query at position m attends to the keys at positions 0..m, itself
 *     included (new tokens are appended before they attend).
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = -1,    /* null pointer, bad size, misaligned buffer   */
  MLA_ERR_UNSUPPORTED = -2,    /* dimensions the library has no kernel for    */
  MLA_ERR_WORKSPACE = -3,      /* workspace or weight buffer too small        */
  MLA_ERR_CUDA = -4,           /* a CUDA runtime call failed                  */
  MLA_ERR_DEVICE_BOUNDS = -5,  /* device-side check: index out of range       */
  MLA_ERR_TIMEOUT = -6         /* device-side bounded wait gave up            */
} mla_status;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype;

typedef struct {
  int n_h;              /* query heads                                       */
  int d_h;              /* per-head content query/key width                  */
  int d_v;              /* per-head value width                              */
  int d_c;              /* KV latent width                                   */
  int d_r;              /* shared RoPE key width (even)                      */
  int d_model;          /* hidden width                                      */
  int d_cq;             /* query latent width; 0 = no query latent           */
  float rope_base;      /* e.g. 10000                                        */
  float softmax_scale;  /* 0 selects 1/sqrt(d_h + d_r) on both score terms   */
  int page_size;        /* tokens per cache page; the library supports 64    */
  mla_dtype dtype;      /* element type of weights, hidden states and cache  */
  int rope_key_per_head; /* 0: one RoPE key shared by all heads (default);
                            1: one d_r key per head (see below)              */
} mla_dims;

/* Per-head RoPE keys (rope_key_per_head = 1).  The 16-head example of "Multi-
 * Head Latent Attention" (talalahmed), "A concrete size comparison", caches
 * one d_r-dim position key per head instead of one shared key: W_KR is then
 * [n_h*d_r, d_model] (rows h*d_r .. for head h), a cache row is
 * [c_t (d_c) | k_R,0,t | ... | k_R,n_h-1,t] (d_c + n_h*d_r values, e.g.
 * 256 + 16*32 = 768 for that example against 288 with a shared key), and head
 * h's position term is q_R,h . k_R,h,t.  The position term is then a per-head
 * contraction rather than part of one dense product over a shared row, so
 * this layout runs on the CUDA-core attention kernel (fp32 and bf16) and
 * needs d_c + n_h*d_r <= 1024; context-parallel decode and the materialised
 * prefill return MLA_ERR_UNSUPPORTED for it. */

/* Opaque host-side handle created by mla_absorb_weights.  It holds the
 * dimensions and pointers into the caller's `absorbed` device buffer. */
typedef struct mla_weights mla_weights;

/* ---------------------------------------------------------------------------
 * Weights.  Absorption (the decoupled-RoPE page's absorption equations) is
 * independent of the cache, so the weight-side layouts are prepared once:
 * W_DKV and W_KR stacked into one [d_c + d_r, d_model] matrix, W_UQ and W_QR
 * stacked into one [n_h*(d_h + d_r), d_in] matrix, each head's W_UK slice
 * transposed to [d_c, d_h], and W_UV and W_DQ copied.  The products with W_UK
 * and W_UV are taken at run time on the query side and after the latent sum.
 * ------------------------------------------------------------------------- */

/* Bytes of device memory mla_absorb_weights needs in `absorbed`; 0 if the
 * dimensions are invalid or unsupported. */
size_t mla_absorbed_weights_bytes(const mla_dims* dims);

/* Copies and re-lays-out the weights into `absorbed` (device, caller-owned,
 * at least mla_absorbed_weights_bytes(dims) bytes, 256-byte aligned) and
 * returns a handle in *out.  W_DQ must be NULL iff dims->d_cq == 0.  The input
 * weights may be freed once the stream has passed this call; `absorbed` must
 * outlive the handle.  Errors: MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED,
 * MLA_ERR_WORKSPACE (buffer too small), MLA_ERR_CUDA. */
mla_status mla_absorb_weights(const mla_dims* dims, const void* W_DKV, const void* W_KR,
                              const void* W_DQ, const void* W_UQ, const void* W_QR,
                              const void* W_UK, const void* W_UV, void* absorbed,
                              size_t absorbed_bytes, mla_weights** out, cudaStream_t stream);

/* Frees the host-side handle (not the caller's device buffer). NULL is a no-op. */
void mla_release_weights(mla_weights* w);

/* Copies the handle's dimensions into *dims. */
mla_status mla_weights_dims(const mla_weights* w, mla_dims* dims);

/* ---------------------------------------------------------------------------
 * Append.  For T tokens with hidden states h [T, d_model], sequence index
 * seq_idx[T] and position pos[T], computes c = W_DKV h and
 * k_R = RoPE_pos(W_KR h) (decoupled-RoPE page; the shared position key of
 * "Latent Attention Meets RoPE") with fp32 accumulation and writes
 * [c | k_R] (rounded to the cache type) into the cache row for (seq, pos).
 * page_table is [num_seqs, max_pages]; a seq_idx outside [0, num_seqs), a
 * position outside [0, max_pages*page_size) or a page id outside
 * [0, num_pages) sets MLA_ERR_DEVICE_BOUNDS in the workspace error word and
 * skips that token's write.
 * Workspace: mla_append_workspace_bytes(dims, T).
 * ------------------------------------------------------------------------- */
size_t mla_append_workspace_bytes(const mla_dims* dims, int T);
mla_status mla_append_latent(const mla_weights* w, const void* h, const int32_t* seq_idx,
                             const int32_t* pos, const int32_t* page_table, int num_seqs,
                             int max_pages, int num_pages, void* cache, int T, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/* Append without a workspace.  The pages have no counterpart to this entry
 * point; it exists for callers that cannot allocate device memory where they
 * append (an engine that owns all of HBM through its own pool, code running
 * under CUDA stream capture, a thread that must not take cudaMalloc's implicit
 * synchronisation).  Same computation and arguments as mla_append_latent,
 * except that the scratch lives in a fixed array inside libmla's own device
 * memory (about 2 MiB, held on every GPU that loads the library until the
 * process exits) and T is limited to MLA_APPEND_NOALLOC_MAX_T tokens; a larger
 * T returns MLA_ERR_WORKSPACE.  It calls no allocating function.
 *   - device_error: optional device int32 (NULL to ignore) into which
 *     MLA_ERR_DEVICE_BOUNDS conditions are OR-ed as the value 1; the caller zeroes
 *     it.
 *   - The first call on a device looks up the array's device address for that
 *     device (with that device current); make that first call before any
 *     stream capture.
 *   - Every call shares the one array and re-zeroes the parts that must start
 *     at zero; calls that can overlap on the GPU (different streams, or
 *     different host threads on one device) race on it and must be serialised
 *     by the caller. */
#define MLA_APPEND_NOALLOC_MAX_T 256
mla_status mla_append_latent_noalloc(const mla_weights* w, const void* h, const int32_t* seq_idx,
                                     const int32_t* pos, const int32_t* page_table, int num_seqs,
                                     int max_pages, int num_pages, void* cache, int T,
                                     int32_t* device_error, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Decode.  B sequences each with n_q new tokens whose hidden states are
 * h_q [B, n_q, d_model]; kv_len[b] (device) counts the keys of sequence b
 * including its n_q new tokens, which must already be appended
 * (mla_append_latent) at positions kv_len[b]-n_q .. kv_len[b]-1.  New token q
 * of sequence b sits at position kv_len[b]-n_q+q and attends to keys
 * 0 .. kv_len[b]-n_q+q.  Writes out [B, n_q, n_h, d_v] as fp32:
 *   q_C, q_R from h (through c_Q = W_DQ h when d_cq > 0),
 *   q~_h = W_UK,h^T q_C,h,  a_t = s*(q~_h . c_t) + s*(RoPE_m(q_R,h) . k_R,t),
 *   alpha = softmax(a),     o_h = W_UV,h sum_t alpha_t c_t.
 * max_kv_len bounds kv_len (host value used for workspace sizing); kv_len[b]
 * outside [n_q, max_kv_len] sets MLA_ERR_DEVICE_BOUNDS and that sequence's
 * outputs are unspecified.  Workspace: mla_decode_workspace_bytes(...).
 * ------------------------------------------------------------------------- */
size_t mla_decode_workspace_bytes(const mla_dims* dims, int B, int n_q, int max_kv_len);
mla_status mla_decode(const mla_weights* w, const void* h_q, const int32_t* kv_len,
                      const int32_t* page_table, int max_pages, int num_pages, const void* cache,
                      float* out, int B, int n_q, int max_kv_len, void* workspace,
                      size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Decode step: append, then decode, in one call.  The same computation as
 * mla_append_latent of the n_q new tokens of every sequence (token q of
 * sequence b at position kv_len[b]-n_q+q, its rows of h as the hidden
 * states) followed by mla_decode with h_q = h: c_KV = W_DKV h and
 * k_R = RoPE(W_KR h) go into `cache` ("ai-decoupled-rope-mla", the cached
 * latent and the decoupled key), then the new tokens attend as in
 * mla_decode.  Outputs and cache rows are bit-identical to the two calls.
 *   - h: [B, n_q, d_model] hidden states of the new tokens.
 *   - kv_len [B] (device): keys per sequence including the new tokens;
 *     page_table must map their positions.
 *   - cache is written (the new rows) and read.
 * With bf16 the append's GEMM runs on the library's side stream (forked from
 * and joined back into `stream` inside the call, as the schedule does) on a
 * share of the SMs, beside the query projections, so it costs little of the
 * step.  Workspace: mla_decode_step_workspace_bytes(...) (the decode
 * workspace plus the append's own split-K scratch).
 * ------------------------------------------------------------------------- */
size_t mla_decode_step_workspace_bytes(const mla_dims* dims, int B, int n_q, int max_kv_len);
mla_status mla_decode_step(const mla_weights* w, const void* h, const int32_t* kv_len,
                           const int32_t* page_table, int max_pages, int num_pages, void* cache,
                           float* out, int B, int n_q, int max_kv_len, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Context-parallel decode: one sequence's cache spread over several ranks
 * (GPUs).  The pages do not split a sequence over devices; the split rests
 * on the identity that the softmax denominators of disjoint key sets add up
 * (the absorbed output of "ai-decoupled-rope-mla", absorption equations, is
 * W_UV applied to a softmax-weighted latent sum, which merges exactly).
 *
 * Rank r holds one page-aligned window of each sequence b, positions
 * window_start[b] .. window_start[b] + window_count[b] - 1 (device int32 [B];
 * start a multiple of page_size; count 0 for none), in its own page pool:
 * page_table [B, max_pages] maps the window's i-th page (positions
 * start + i*page_size ..) to a page of `cache`.  Tokens are appended with
 * mla_append_latent at their GLOBAL positions through a table indexed by
 * global page (the window's pages at index start/page_size + i, -1 elsewhere),
 * so the RoPE key carries the global position.
 *
 * mla_decode_cp_partial: for new token q of sequence b (global position
 * kv_len[b]-n_q+q, kv_len the GLOBAL key count) and every head, the attention
 * over the keys of the window at positions <= its own: writes the normalised
 * latent sum obar_out [B, n_q, n_h, d_c] (bf16) and
 * lse_out [B, n_q, n_h] (fp32) = log2 sum_t exp(a_t) over those keys; a row
 * with no such key gets lse = -inf and an unspecified obar row.  A window that
 * is negative, not page-aligned or longer than max_pages*page_size sets
 * MLA_ERR_DEVICE_BOUNDS and counts as empty.
 *
 * mla_decode_cp_combine: merges every rank's partials, obar_parts
 * [n_ranks, B, n_q, n_h, d_c] (bf16) and lse_parts [n_ranks, B, n_q, n_h]
 * (fp32), as obar = sum_r 2^(lse_r - L) obar_r with L = log2 sum_r 2^lse_r,
 * then writes out [B, n_q, n_h, d_v] (fp32) = W_UV,h obar_h.  A row that no
 * rank saw sets MLA_ERR_DEVICE_BOUNDS and yields zeros.  The exchange of the
 * partials between ranks (an all-gather) is the caller's.
 *
 * bf16 only (an fp32 mla_dims returns MLA_ERR_UNSUPPORTED).  Both calls take
 * a workspace of mla_decode_cp_workspace_bytes(dims, B, n_q).
 * ------------------------------------------------------------------------- */
size_t mla_decode_cp_workspace_bytes(const mla_dims* dims, int B, int n_q);
mla_status mla_decode_cp_partial(const mla_weights* w, const void* h_q, const int32_t* kv_len,
                                 const int32_t* window_start, const int32_t* window_count,
                                 const int32_t* page_table, int max_pages, int num_pages,
                                 const void* cache, void* obar_out, float* lse_out, int B, int n_q,
                                 int max_kv_len, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream);
mla_status mla_decode_cp_combine(const mla_weights* w, int n_ranks, const void* obar_parts,
                                 const float* lse_parts, float* out, int B, int n_q,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Causal prefill on the absorbed path.  h [B, S, d_model]: token s of
 * sequence b sits at position s.  Appends all B*S tokens to the cache (the
 * page table must cover S positions per sequence), then every token attends
 * to positions <= its own.  Writes out [B, S, n_h, d_v] fp32.
 * Workspace: mla_prefill_workspace_bytes(dims, B, S).
 * ------------------------------------------------------------------------- */
size_t mla_prefill_workspace_bytes(const mla_dims* dims, int B, int S);
mla_status mla_prefill(const mla_weights* w, const void* h, const int32_t* page_table,
                       int max_pages, int num_pages, void* cache, float* out, int B, int S,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Causal prefill in the materialised form ("Multi-Head Latent Attention"
 * (talalahmed), "Compress first, expand later" and its closing flow diagram):
 * the same result as mla_prefill, computed by expanding every token's latent
 * into per-head keys K_C = W_UK,h c_t and values V = W_UV,h c_t and running
 * causal multi-head attention on [K_C | k_R] (d_h + d_r columns) and V, so the
 * output needs no W_UV after the sum.  It does 2 (d_h + d_r) + 2 d_v flops
 * per (query, key) pair and head instead of 2 (d_c + d_r) + 2 d_c, at the cost
 * of writing and reading the expanded K_C and V.  Absorbed and materialised
 * results agree to rounding, not bit for bit (the order of the products
 * differs; "ropeabsorb", "Absorption is exact").
 * Arguments, layouts and the cache append are those of mla_prefill.  Supports
 * bf16 with d_r = 64, d_h in {64, 128} and d_v in {64, 128}; other dimensions
 * return MLA_ERR_UNSUPPORTED (the size query returns 0).
 * Workspace: mla_prefill_materialised_workspace_bytes(dims, B, S) (it holds the
 * expanded K_C and V: 2 * B * S * n_h * (d_h + d_v) bytes of it).
 * ------------------------------------------------------------------------- */
size_t mla_prefill_materialised_workspace_bytes(const mla_dims* dims, int B, int S);
mla_status mla_prefill_materialised(const mla_weights* w, const void* h, const int32_t* page_table,
                                    int max_pages, int num_pages, void* cache, float* out, int B,
                                    int S, void* workspace, size_t workspace_bytes,
                                    cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Status.
 * ------------------------------------------------------------------------- */
/* Waits for `stream`, then returns the error recorded on the device by the
 * most recent call that used `workspace` (MLA_OK if none): MLA_ERR_TIMEOUT
 * (a bounded wait gave up), MLA_ERR_DEVICE_BOUNDS (a page id or length out
 * of range), or MLA_ERR_UNSUPPORTED (the device placed the attention
 * kernel's shared memory off the 1024-byte alignment it relies on). */
mla_status mla_get_error(const void* workspace, cudaStream_t stream);

/* Test hook for the failure path (the pages have no counterpart).  Launches
 * one warp that waits, bounded by limit_us microseconds, on an mbarrier that
 * nothing ever arrives at.  When the bound runs out the wait records
 * MLA_ERR_TIMEOUT in the error word of `workspace` exactly as the library's
 * pipelined kernels do on a stalled pipeline, and the kernel returns; no copy
 * or MMA is in flight, so the context stays usable.  mla_get_error(workspace)
 * then reports MLA_ERR_TIMEOUT.  workspace: device memory of at least 256
 * bytes, 256-byte aligned; its error word is zeroed first.  Errors:
 * MLA_ERR_INVALID_ARG (null or misaligned workspace, limit_us outside
 * [1, 1000000]), MLA_ERR_CUDA. */
mla_status mla_selftest_wait_timeout(void* workspace, int limit_us, cudaStream_t stream);

/* Static, human-readable name of a status code. */
const char* mla_status_string(mla_status s);

/* Number of kernel launches the most recent call on this host thread issued
 * (for launch accounting in benchmarks). */
int mla_last_launch_count(void);

/* Kernel timing for benchmarks.  Between mla_profile_begin and
 * mla_profile_end, every launch of the latent-attention kernel (the step that
 * streams the cache) made on this host thread is bracketed by a pair of CUDA
 * events recorded on the call's stream; at most max_launches launches are
 * timed.  mla_profile_end waits for the last event and returns the summed
 * kernel time in milliseconds and the number of timed launches.  Creates CUDA
 * events (no device memory).  Errors: MLA_ERR_INVALID_ARG, MLA_ERR_CUDA. */
mla_status mla_profile_begin(int max_launches);
mla_status mla_profile_end(double* total_ms, int* launches);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H_ */
