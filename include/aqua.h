/*
 * aqua.h -- C ABI of the B200 (sm_100a) library for AQUA's online attention step.
 *
 * AQUA (Attention via QUery mAgnitudes, arXiv 2509.11155): an orthogonal d x d
 * projection P is computed once offline from an SVD of calibration queries and
 * keys; online, every query and key is projected (q~ = qP, k~ = kP), each query
 * head keeps the k dimensions where |q~| is largest (ties to the lower index),
 * scores are computed on those dimensions only (scaled by 1/sqrt(d)), followed
 * by softmax and the weighted sum of the unprojected values.  Sources: the
 * paper's abstract; edgentiq blog "How AQUA Works: A Two-Phase Approach" and
 * "AQUA-Memory: Dual Savings" (statically truncated cache); H2O eviction is
 * named in the abstract (AQUA combines with token eviction methods such as H2O
 * and speeds them up).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers unless stated otherwise, owned by
 *     the caller, 16-byte aligned, dense row-major in the layout given.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; 0 = legacy
 *     default stream).  No entry point allocates or frees device memory and no
 *     entry point synchronises the stream.  Scratch space is caller-provided
 *     (`workspace`, size from the matching *_workspace_size call).
 *   - Return value: AQUA_OK or a negative status.  On a negative status nothing
 *     was enqueued (argument errors are detected on the host before any launch),
 *     except AQUA_ERR_CUDA, which reports a failed launch.  aqua_last_error()
 *     returns a thread-local message describing the last failure.
 *   - Device-side waits are bounded (about 2 s); a wait that runs out records
 *     AQUA_ERR_TIMEOUT in the cache's status word (read by aqua_status) and the
 *     kernel returns early instead of hanging.
 *   - head_dim d must be 128.
 */
#ifndef AQUA_H_
#define AQUA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AQUA_API __attribute__((visibility("default")))
#else
#define AQUA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* aqua_stream_t; /* identical to cudaStream_t */

enum aqua_status_code {
  AQUA_OK = 0,
  AQUA_ERR_ARG = -1,         /* bad argument (null pointer, size out of range, misalignment) */
  AQUA_ERR_UNSUPPORTED = -2, /* shape or dtype this build does not implement */
  AQUA_ERR_WORKSPACE = -3,   /* workspace smaller than the *_workspace_size result */
  AQUA_ERR_CUDA = -4,        /* a CUDA call or launch failed */
  AQUA_ERR_TIMEOUT = -5      /* a bounded device-side wait ran out (reported by aqua_status) */
};

enum aqua_dtype { AQUA_F32 = 0, AQUA_BF16 = 1 };

/* Number of int32 control words the cache's `ctrl` buffer must hold. */
#define AQUA_CTRL_WORDS 16

/*
 * The KV cache descriptor.  The struct itself is host memory owned by the
 * caller; the buffers it points to are device memory owned by the caller.
 *
 *   k_proj  [B][Hkv][d_store][Tcap]  dtype  projected keys k~ = kP, DIMENSION-MAJOR:
 *                                           row j of (b, g) holds dimension j of
 *                                           every cached token, contiguous over
 *                                           tokens.  d_store = m < d keeps only the
 *                                           first m projected dimensions
 *                                           (AQUA-Memory static truncation).
 *   v       [B][Hkv][Tcap][dv]       dtype  values, token-major.  dv_store = 0: the
 *                                           unprojected values (dv = d).  dv_store > 0
 *                                           (AQUA-Memory on the values): the first
 *                                           dv = dv_store dimensions of v P, the
 *                                           projected value; outputs are brought back
 *                                           as o = o^ P[:, :dv_store]^T.
 *   len     [B]                      int32  tokens (slots) in use per sequence.
 *   n_abs   [B]                      int32  tokens ever appended per sequence (the
 *                                           absolute position of the next token);
 *                                           nullable unless pos != NULL.
 *   pos     [B][Hkv][Tcap]           int32  nullable; absolute position held by each
 *                                           slot (required for H2O eviction).
 *   score   [B][Hkv][Tcap]           f32    nullable; H2O cumulative attention score
 *                                           of each slot.
 *   ctrl    [AQUA_CTRL_WORDS]        int32  control words; must be zero when the
 *                                           cache is created; the library leaves
 *                                           them zero except the sticky status
 *                                           word read by aqua_status.
 *   max_len  host int: an upper bound of every len[b]; aqua_project_keys adds L,
 *            aqua_h2o_update lowers it to the budget.
 *   dv_store host int: 0, or the number of projected value dimensions stored
 *            (a multiple of 16, at most d).  The edgentiq blog ("AQUA-Memory:
 *            Dual Savings") drops the lowest-importance dimensions of both keys
 *            and values before caching; the reading taken: values use the KV
 *            head's P like the keys and the first dv_store projected dimensions
 *            are kept.  Prefill requires dv_store = 0.
 *   Tcap must be a multiple of 16; dtype is AQUA_BF16 or AQUA_F32 for both k_proj and v.
 */
typedef struct aqua_cache {
  void* k_proj;
  void* v;
  int32_t* len;
  int32_t* n_abs;
  int32_t* pos;
  float* score;
  int32_t* ctrl;
  int B, Hkv, d, d_store, Tcap;
  int max_len;
  int dtype;
  int dv_store;
} aqua_cache;

/* Thread-local text of the last failure on this host thread ("" if none). */
AQUA_API const char* aqua_last_error(void);

/* Library ABI version (increments when a signature changes). */
AQUA_API int aqua_version(void);

/*
 * Reads and clears the sticky device status word of `cache` (synchronises
 * `stream`).  *status_out receives AQUA_OK or the first device-side error
 * (AQUA_ERR_TIMEOUT).  Returns AQUA_OK unless the copy itself failed.
 */
AQUA_API int aqua_status(const aqua_cache* cache, int* status_out, aqua_stream_t stream);

/*
 * Offline calibration (abstract: one projection matrix, computed offline
 * by an SVD of calibration data and shared across languages; edgentiq, "Offline Projection
 * Computation").  X [n][d] f32 stacks calibration queries and keys (not
 * centred).  Writes P [d][d] f32 whose COLUMNS are the right singular vectors
 * of X ordered by descending singular value, and sigma [d] f32.  Each column's
 * largest-magnitude entry is made positive.  Computed on the GPU: the Gram
 * matrix X^T X in f64, then cyclic Jacobi eigen-decomposition in f64.
 * Requires 1 <= n, d == 128.
 */
AQUA_API size_t aqua_calibrate_workspace_size(int n, int d);
AQUA_API int aqua_calibrate(const float* X, int n, int d, float* P_out, float* sigma_out,
                   void* workspace, size_t workspace_bytes, aqua_stream_t stream);

/*
 * Key projection and append (abstract: queries and keys are projected by P;
 * edgentiq, "Online Inference").  For every sequence b and new token l < L:
 * k~ = k_new[b][l][g] . P[g] is computed in f32, its first d_store dimensions
 * are rounded to the cache dtype (bf16: round-to-nearest-even) and written into
 * slot len[b] + l of k_proj (dimension-major); v_new is copied into the same
 * slot of v (with dv_store > 0: v~ = v_new P[g] in f32, its first dv_store
 * dimensions rounded to the cache dtype).  If pos/score are present the slot's position is n_abs[b] + l and
 * its score 0.  Afterwards len[b] += L and n_abs[b] += L on the device, and
 * cache->max_len += L on the host.
 *   k_new, v_new  [B][L][Hkv][d]  cache dtype
 *   P             [Hkv][d][d]     f32, q~ = q P (row vector times P)
 * k_new, v_new and P are read before the call waits for the preceding kernel
 * on the stream (the lengths and the cache only after it), which is safe
 * unless the kernel that wrote them released its dependents early through
 * programmatic dependent launch (no kernel here that writes them does).
 * Errors: AQUA_ERR_ARG if cache->max_len + L > Tcap or L < 1.
 */
AQUA_API int aqua_project_keys(aqua_cache* cache, const void* k_new, const void* v_new, const float* P,
                      int L, aqua_stream_t stream);

/*
 * One decode step of AQUA attention for every sequence and query head, over
 * the len[b] cached tokens.  It follows the online phase of the method
 * (abstract: queries and keys are projected, a sparse subset of dimensions is
 * chosen by the query's magnitude, the attention scores use only those
 * dimensions; edgentiq, "How AQUA Works: A Two-Phase Approach", Online
 * Inference): q~ = q P; S_h = the k dimensions with the largest |q~_j| (ties
 * to the lower index); s_t = sum over j in S_h of q~_j k~_t[j] / sqrt(d);
 * softmax over the visible tokens; o_h = sum_t p_t v_t over the unprojected
 * values.  The 1/sqrt(d) scale, the tie rule and the unprojected V are the
 * workload statement's readings where the pages are silent.
 *   q          [B][Hq][d]  cache dtype; query head h uses KV head h / (Hq/Hkv)
 *   k_new, v_new  nullable [B][Hkv][d] cache dtype: the step's new key and
 *              value.  When given they are appended, exactly as
 *              aqua_project_keys(cache, k_new, v_new, P, 1) would (slot len[b],
 *              len[b] += 1, cache->max_len += 1), and the step attends them
 *              (len[b] + 1 tokens).  On the device len[b] and n_abs[b] advance
 *              when the step's last kernel finishes.  When NULL the caller
 *              appended the step's key beforehand.
 *   P          [Hkv][d][d] f32.  P (and, when B*Hkv exceeds the SM count,
 *              q) are read before the step waits for the preceding kernel on
 *              the stream, which is safe unless the kernel that wrote them
 *              released its dependents early through programmatic dependent
 *              launch (no kernel here that writes them does).
 *   k          dimensions kept per query head, 1 <= k <= d_store
 *   scale      score scale; <= 0 selects 1/sqrt(d) (d = full head dim)
 *   out        [B][Hq][d]  out_dtype (AQUA_F32 or AQUA_BF16, RNE)
 *   sel_out    nullable [B][Hq][k] int32: selected dimensions, ascending
 *   qproj_out  nullable [B][Hq][d] f32: the projected query q~ the selection used
 *   scores_out nullable [B][Hq][Tcap] f32: score of every cached slot (scaled)
 *   lse_out    nullable [B][Hq] f32: log-sum-exp of the scores
 *   workspace  device, 256-byte aligned, >= aqua_decode_workspace_size bytes;
 *              caller-owned scratch, contents need no initialisation.  Its
 *              selection buffers have two halves; successive calls on one
 *              workspace alternate between them (tracked per workspace
 *              address), so a step's selection can be written while the
 *              previous step's attention kernel still reads the other half.
 * Hq must be a multiple of Hkv with Hq/Hkv in {1, 2, 4}.  A sequence with
 * len[b] = 0 gets a zero output and lse = -inf.
 * Errors: AQUA_ERR_ARG if only one of k_new, v_new is given or the cache is full.
 */
AQUA_API size_t aqua_decode_workspace_size(const aqua_cache* cache, int Hq);
AQUA_API int aqua_decode_attn(aqua_cache* cache, const void* q, const void* k_new, const void* v_new,
                              const float* P, int Hq, int k, float scale, void* out, int out_dtype,
                              int32_t* sel_out, float* qproj_out, float* scores_out, float* lse_out,
                              void* workspace, size_t workspace_bytes, aqua_stream_t stream);

/*
 * The decode step of aqua_decode_attn as two calls on the same stream, which
 * together enqueue exactly the two kernels aqua_decode_attn enqueues and give
 * bit-identical results:
 *   aqua_decode_select  the online selection (abstract: project the query, pick
 *                       the dimensions by the query's magnitude): q~ = q P,
 *                       top-k of |q~| per query head, the group's union of
 *                       kept dimensions and the masked queries, written to the
 *                       workspace; with k_new/v_new also the append (slot
 *                       len[b], cache->max_len += 1; len[b] itself advances at
 *                       the end of aqua_decode_attend).
 *   aqua_decode_attend  the sparse-dimension attention over that selection
 *                       (edgentiq, "How AQUA Works", Online Inference: scores
 *                       on the selected dimensions, softmax, weighted sum of
 *                       the values), split over the SMs and merged.
 * Use: a caller that wants to schedule or time the two halves separately (an
 * event between them serialises the second behind the first; back to back
 * they overlap as in aqua_decode_attn).  The workspace carries the selection
 * from the first call to the second; neither it nor the cache may be touched
 * in between.  `appended` must be 1 exactly when the preceding
 * aqua_decode_select was given k_new/v_new.  P may be NULL for
 * aqua_decode_attend unless cache->dv_store > 0 (the output's back-projection
 * reads it).  Arguments as aqua_decode_attn;
 * each call checks the arguments it uses (AQUA_ERR_ARG for appended not 0/1,
 * or 1 with an empty cache).
 */
AQUA_API int aqua_decode_select(aqua_cache* cache, const void* q, const void* k_new, const void* v_new,
                                const float* P, int Hq, int k, float scale, int32_t* sel_out, float* qproj_out,
                                void* workspace, size_t workspace_bytes, aqua_stream_t stream);
AQUA_API int aqua_decode_attend(aqua_cache* cache, const float* P, int Hq, int appended, void* out,
                                int out_dtype, float* scores_out, float* lse_out, void* workspace,
                                size_t workspace_bytes, aqua_stream_t stream);

/*
 * The decode step of aqua_decode_attn for callers that cannot provide device
 * scratch memory: their device memory belongs to another allocator they may
 * not bypass with cudaMalloc (a framework pool, a fixed memory budget), or
 * their interface has no place for a workspace buffer.  The paper has no
 * counterpart to this entry point; it is an interface convenience.
 *   - Arguments and results as aqua_decode_attn, without workspace and
 *     workspace_bytes.  Nothing is allocated or freed.
 *   - The scratch is an 8 MiB array inside the library's device image; every
 *     GPU that loads the library keeps it until the library is unloaded.
 *     AQUA_ERR_WORKSPACE if the shape needs more (aqua_decode_workspace_size
 *     gives the need); nothing is launched then.
 *   - The first call on a device looks up the array's address on that device;
 *     make that first call before any stream capture.
 *   - All calls share the array, which keeps the previous call's contents; the
 *     kernels re-initialise what they depend on.  Calls that overlap on the GPU
 *     (e.g. on two streams) race on it and must be ordered by the caller.
 */
AQUA_API int aqua_decode_attn_static(aqua_cache* cache, const void* q, const void* k_new, const void* v_new,
                                     const float* P, int Hq, int k, float scale, void* out, int out_dtype,
                                     int32_t* sel_out, float* qproj_out, float* scores_out, float* lse_out,
                                     aqua_stream_t stream);

/*
 * Causal AQUA attention for a chunk of L prompt tokens at absolute positions
 * pos0 .. pos0+L-1 of every sequence (their keys must already be appended, so
 * len[b] >= pos0 + L).  Row i of sequence b attends to slots 0 .. pos0+i; each
 * (row, head) selects its own k dimensions; the dimension-masked Q K~^T and
 * P V run on the tensor cores.  The pages describe only the per-query step
 * (abstract; edgentiq, "How AQUA Works", Online Inference); chunked causal
 * prefill applies that step to every prompt row, as the workload statement's
 * prefill configuration (a 4096-token prompt in 512-token chunks, causal)
 * asks.  Row i's result equals a decode step at position pos0+i.
 *   q    [B][L][Hq][d] cache dtype (bf16 only)
 *   out  [B][L][Hq][d] out_dtype
 *   sel_out   nullable [B][L][Hq][k] int32: selected dimensions, ascending
 *   qproj_out nullable [B][L][Hq][d] f32: the projected queries q~ the selection
 *             used (computed on the tensor cores with P split into three bf16
 *             parts, f32 accumulation), 16-byte aligned
 *   workspace  device, 256-byte aligned, >= aqua_prefill_workspace_size bytes
 *              (a small reserved block: projection, selection and attention
 *              run in one kernel and keep their intermediates on chip)
 * Requires Hq/Hkv in {1, 2, 4}, d_store a multiple of 16, k <= d_store.
 * A wait that exceeds its time limit inside the kernel records
 * AQUA_ERR_TIMEOUT in the cache's status word (aqua_status).
 */
AQUA_API size_t aqua_prefill_workspace_size(const aqua_cache* cache, int Hq, int L);
AQUA_API int aqua_prefill_attn(const aqua_cache* cache, const void* q, int pos0, int L, const float* P,
                      int Hq, int k, float scale, void* out, int out_dtype, int32_t* sel_out, float* qproj_out,
                      void* workspace, size_t workspace_bytes, aqua_stream_t stream);

/*
 * H2O heavy-hitter update after a decode step (abstract: AQUA accelerates
 * token eviction methods like H2O).  Reading of the rule: for every (b, KV
 * head g) and slot t < len[b], score[t] += sum over the group's query heads h
 * of exp(scores[b][h][t] - lse[b][h]) (the AQUA softmax probabilities from
 * aqua_decode_attn).  Then, if len[b] > budget, exactly one slot is evicted
 * per (b, g): the lowest score among slots whose position is at most
 * newest - recent (newest = n_abs[b] - 1), ties to the smaller position; the
 * last slot is moved into its place and len[b] becomes len[b] - 1.
 *   scores [B][Hq][Tcap], lse [B][Hq]  from aqua_decode_attn
 *   evicted_out nullable [B][Hkv] int32: evicted absolute position, or -1
 * Requires pos, score and n_abs in the cache and Hq/Hkv in {1, 2, 4}
 * (AQUA_ERR_UNSUPPORTED otherwise, nothing launched).  cache->max_len is
 * lowered to min(max_len, budget) on the host.
 */
AQUA_API int aqua_h2o_update(aqua_cache* cache, const float* scores, const float* lse, int Hq, int budget,
                    int recent, int32_t* evicted_out, aqua_stream_t stream);

/*
 * Diagnostic: launches one CTA that waits, with the bounded wait every kernel
 * of the library uses, on a barrier that is never completed, for limit_ns
 * nanoseconds (1 us .. 2 s); the wait runs out, the kernel records
 * AQUA_ERR_TIMEOUT in the cache's status word (read it with aqua_status) and
 * returns.  It lets a caller check the time-out path on its GPU: nothing
 * faults or hangs and the context stays usable.  The paper has no counterpart.
 * Errors: AQUA_ERR_ARG for a missing ctrl block or a limit outside the range.
 */
AQUA_API int aqua_selftest_wait_timeout(aqua_cache* cache, unsigned long long limit_ns, aqua_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* AQUA_H_ */
