/*
 * hs2.h -- C ABI of libhs2, the B200 (sm_100a) hot path of the HySparse2
 * Cross-Decoder hybrid block.
 *
 * The HySparse2 pages describe a model split into a Self-Decoder and a
 * Cross-Decoder joined by two levels of KV sharing (IT Home announcement of
 * MiMo HySparse2, the "KV Bridging" / "KV Reuse" paragraphs; toolnavs.com
 * summary, section "HySparse2 がやったこと"):
 *   1. KV Bridging: every full-attention layer of the Cross-Decoder builds its
 *      own K/V cache from the input hidden state of the corresponding
 *      Self-Decoder full-attention layer, with its own K/V projection.
 *   2. KV Reuse: inside a hybrid block (one full-attention layer followed by
 *      several sparse-attention layers), the full-attention layer selects
 *      important positions from its attention scores while it computes, and
 *      the sparse layers reuse its KV cache and those indices.
 *   Selection is per token: the 128 most recent tokens are always taken, and
 *   1024 global tokens are chosen from outside that window (IT Home
 *   announcement, token-level selection paragraph; cnyes.com article, section
 *   "檢索精確到token").
 *
 * The three compute entry points below are those three steps.  The pages give
 * no formulas; the readings this library takes are stated at each function.
 *
 * Conventions (all functions):
 *   - Every tensor pointer is a DEVICE pointer owned by the caller.  The
 *     library allocates no device or host memory; scratch comes from the
 *     caller's workspace, sized by the matching *_workspace() function.
 *   - Work is enqueued on `stream` and the call returns without waiting.
 *     Arguments are checked on the host before anything is enqueued; a bad
 *     argument returns HS2_ERR_INVALID_ARG and enqueues nothing.  A shape the
 *     kernels do not implement returns HS2_ERR_UNSUPPORTED.  A failed launch
 *     returns HS2_ERR_CUDA.  The library never aborts or exits.
 *   - Kernels that wait on on-chip barriers give up after about one second,
 *     set a bit in a per-device status word and return; read and clear it
 *     with hs2_last_device_status().
 *   - Pointers must be 16-byte aligned.  bf16 is IEEE binary32's upper half;
 *     E4M3 is the OCP 8-bit float (bias 7, max 448, no infinities).
 *   - MQA cache layout: one KV head.  For B sequences of L positions, K and V
 *     are [B][L][D] row-major (bf16: 2 bytes, E4M3: 1 byte per element); for
 *     E4M3, k_scale and v_scale are fp32 [B][L] and the stored value of
 *     element d of position j is e4m3(code) * scale[j].
 */
#ifndef HS2_H
#define HS2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HS2_API __attribute__((visibility("default")))
#else
#define HS2_API
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* hs2_stream_t;

typedef enum {
  HS2_OK = 0,
  HS2_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, inconsistent sizes  */
  HS2_ERR_UNSUPPORTED = 2,  /* valid request, shape not implemented         */
  HS2_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed         */
  HS2_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than required      */
  HS2_ERR_TIMEOUT = 5,      /* a kernel gave up waiting on a barrier        */
  HS2_ERR_DEVICE = 6        /* a kernel found an out-of-range index         */
} hs2_status;

typedef enum { HS2_KV_BF16 = 0, HS2_KV_FP8_E4M3 = 1 } hs2_kv_dtype;

/* One layer's MQA cache: device pointers.  Scales are NULL for bf16. */
typedef struct {
  void* k;
  void* v;
  float* k_scale;
  float* v_scale;
} hs2_kv_cache;

/*
 * hs2_bridge_kv -- KV Bridging (IT Home announcement, "KV Bridging"
 * paragraph; toolnavs.com summary: each target layer has its own K/V
 * projection of the same source hidden state).
 *
 * For every target layer l in [0, n_layers) and token r in [0, T):
 *   K_l[r][d] = sum_k X[r][k] * Wt[l*2*D + d][k]
 *   V_l[r][d] = sum_k X[r][k] * Wt[l*2*D + D + d][k]
 * computed as one GEMM Y = X * Wt^T with fp32 accumulation.
 *   X   : bf16 [T][hidden] row-major (the source layer's input hidden state).
 *   Wt  : bf16 [n_layers*2*D][hidden] row-major; row c holds the weights of
 *         output column c (nn.Linear weight layout).
 *   caches[l] (host array of n_layers structs of device pointers): rows
 *         cache_row_offset .. cache_row_offset+T-1 of K_l and V_l are written.
 *   out_dtype HS2_KV_BF16: K, V bf16 [rows][D] (round to nearest even).
 *   out_dtype HS2_KV_FP8_E4M3: per token and tensor, s = max_d |Y| / 448
 *         (s = 1 when the row is all zero) is written to k_scale/v_scale[row]
 *         and the codes E4M3(Y / s) (round to nearest even, saturating) to
 *         K/V [rows][D].
 * Supported: D == 128, hidden % 64 == 0, hidden >= 64, n_layers >= 1.
 */
HS2_API hs2_status hs2_bridge_kv(const void* X, int64_t T, int hidden, const void* Wt, int n_layers,
                         int D, hs2_kv_dtype out_dtype, const hs2_kv_cache* caches,
                         int64_t cache_row_offset, hs2_stream_t stream);

/*
 * Workspace bytes needed by hs2_full_attn_select for these sizes.
 * Returns 0 for arguments hs2_full_attn_select would reject.
 */
HS2_API size_t hs2_full_attn_select_workspace(int B, int T, int64_t L, int H, int D, int topk,
                                      int window, hs2_kv_dtype dt);

/*
 * hs2_full_attn_select -- the hybrid block's full-attention layer and its
 * token selection (IT Home announcement, "KV Reuse" paragraphs: the full
 * layer picks important positions from its attention scores; token-level
 * selection paragraph: 128 most recent tokens forced, 1024 more from outside
 * that window).
 *
 * Query t of sequence b sits at position i = L - T + t of that sequence's
 * cache (the cache already holds the queries' own tokens).  For head h:
 *   s_hj   = scale * <Q[b][t][h], K[b][j]>          for j <= i (causal)
 *   p_hj   = exp(s_hj - lse_h),  lse_h = log sum_{j<=i} exp(s_hj)
 *   O[b][t][h][d] = sum_j p_hj V[b][j][d]
 * Selection (readings of this library where the pages are silent):
 *   score_j = sum_h p_hj (head-summed softmax probability);
 *   candidates C = {0 .. i-window}; window W = {max(0,i-window+1) .. i};
 *   S = W  union  the min(topk, |C|) candidates of largest score, ties to
 *   the lower position.
 * Outputs:
 *   O     : fp32 [B][T][H][D].
 *   lse   : fp32 [B][T][H] natural-log normaliser, or NULL.
 *   idx   : int32 [B][T][topk+window]: S in ascending order, then -1 padding.
 *   n_sel : int32 [B][T]: |S| = min(topk, |C|) + min(window, i+1).
 * Inputs: Q bf16 [B][T][H][D]; kv points to one hs2_kv_cache (host struct).
 * Supported: D in {64, 128}; H in {8, 16, 32}; 1 <= T <= L; L < 2^31;
 * 0 <= topk; 1 <= window; topk + window <= 4096.
 */
HS2_API hs2_status hs2_full_attn_select(const void* Q, const hs2_kv_cache* kv, int B, int T, int64_t L,
                                int H, int D, float scale, int topk, int window,
                                hs2_kv_dtype dt, float* O, float* lse, int32_t* idx,
                                int32_t* n_sel, void* workspace, size_t workspace_bytes,
                                hs2_stream_t stream);

/*
 * hs2_full_attn_select_blocks -- hs2_full_attn_select with the block-level
 * selection of the HySparse generation before HySparse2, for comparison with
 * the token-level selection (dpshk.com explainer, section 03: history chosen
 * in blocks of 64 tokens, so a block with one useful token takes the budget
 * of 64; cnyes.com article, section "檢索精確到token": the ablation keeps the
 * same budget and compares the two granularities).
 *
 * O and lse are those of hs2_full_attn_select.  Selection (readings of this
 * library where the pages are silent): candidates C = {0 .. i-window} as for
 * tokens; block b = positions b*block .. b*block+block-1, a candidate when it
 * holds a candidate position; its score is the sum of score_j over its
 * candidate positions; the topk/block blocks of largest score are kept, ties
 * to the lower block; S = their candidate positions union the window,
 * ascending in idx[b][t][0 .. n_sel), then -1.  When no more than topk/block
 * blocks are candidates, S = {0 .. i}.  |S| <= topk + window.
 * Arguments, layouts, workspace (hs2_full_attn_select_workspace) and status
 * codes are those of hs2_full_attn_select, plus: block >= 1 and topk a
 * multiple of block (else HS2_ERR_INVALID_ARG); at most 49152 candidate blocks
 * per query, (L - window) / block + 1 <= 49152 (else HS2_ERR_UNSUPPORTED).
 */
HS2_API hs2_status hs2_full_attn_select_blocks(const void* Q, const hs2_kv_cache* kv, int B, int T,
                                               int64_t L, int H, int D, float scale, int topk,
                                               int window, int block, hs2_kv_dtype dt, float* O,
                                               float* lse, int32_t* idx, int32_t* n_sel,
                                               void* workspace, size_t workspace_bytes,
                                               hs2_stream_t stream);

/*
 * Context parallelism of the full-attention layer and its selection: G ranks
 * (one per GPU) each hold a contiguous slice of every sequence's cache, L_r
 * positions starting at global position a_r, and all T queries (query t at
 * global position q_pos0 + t; a slice-relative position q_pos0 + t - a_r).  The
 * pages analyse contexts of a million tokens (dpshk.com explainer, section 05;
 * cnyes.com article, cost paragraph), where one layer's cache spans devices.
 * One layer is, on every rank:
 *   1. hs2_cp_attn_partial   -> O_r (normalised over the slice), lse_r
 *   2. all-gather of lse_r, hs2_cp_lse_combine -> lse (global normaliser)
 *   3. hs2_cp_rescale(O_r), sum all-reduce of O_r across ranks -> O
 *   4. hs2_cp_select_local   -> the slice's top-k candidates and their scores
 *   5. all-gather of the candidate lists, hs2_cp_merge_select -> idx, n_sel
 * The results equal hs2_full_attn_select on the whole cache (same readings):
 * the global top-k lies in the union of the slices' top-k lists, and the
 * merge keeps ties at the lower position.  The collectives are the caller's
 * (NCCL through torch.distributed in the Python package).  Supported: D ==
 * 128, H in {8, 16, 32}, B * L_r < 2^31; T may exceed L_r.
 *
 * Workspace bytes of hs2_cp_attn_partial / hs2_cp_select_local on one slice;
 * 0 for arguments they would reject.
 */
HS2_API size_t hs2_cp_workspace(int B, int T, int64_t L_local, int H, int D, int topk, int window,
                                hs2_kv_dtype dt);

/*
 * Step 1 on one slice: kv holds the slice, K/V [B][L_local][D]; q_pos_local is
 * query 0's slice-relative position (global position - a_r; it may be
 * negative or >= L_local).  Key j of the slice is visible to query t when
 * j <= q_pos_local + t.  Writes O fp32 [B][T][H][D] (normalised over the
 * visible keys of the slice; 0 where none is visible) and lse fp32 [B][T][H]
 * (natural log; -inf where none is visible).
 */
HS2_API hs2_status hs2_cp_attn_partial(const void* Q, const hs2_kv_cache* kv, int B, int T,
                                       int64_t L_local, int64_t q_pos_local, int H, int D,
                                       float scale, hs2_kv_dtype dt, float* O, float* lse,
                                       void* workspace, size_t workspace_bytes,
                                       hs2_stream_t stream);

/*
 * Step 2: lse[e] = log sum_r exp(lse_parts[r * n + e]) for e < n (lse_parts
 * fp32 [G][n], -inf entries contribute nothing).
 */
HS2_API hs2_status hs2_cp_lse_combine(const float* lse_parts, int G, int64_t n, float* lse,
                                      hs2_stream_t stream);

/*
 * Step 3 (before the sum across ranks): O_part[e][d] *= exp(lse_part[e] -
 * lse[e]) for the n rows of D values (0 where lse_part is -inf).
 */
HS2_API hs2_status hs2_cp_rescale(float* O_part, const float* lse_part, const float* lse,
                                  int64_t n, int D, hs2_stream_t stream);

/*
 * Step 4 on one slice: with lse the global normaliser (step 2's output,
 * [B][T][H]), score_j = sum_h exp(s_hj - lse_h) for the slice's candidates
 * (slice-relative j <= q_pos_local + t - window, j < L_local), and the slice's
 * top-k of them by (score descending, position ascending): cand_idx int32
 * [B][T][topk] global positions (slice position + key_pos0, key_pos0 = a_r),
 * ascending, -1 padded; cand_score fp32 [B][T][topk] their scores (-1 for
 * padding).  topk >= 1.
 */
HS2_API hs2_status hs2_cp_select_local(const void* Q, const hs2_kv_cache* kv, int B, int T,
                                       int64_t L_local, int64_t q_pos_local, int64_t key_pos0,
                                       int H, int D, float scale, int topk, int window,
                                       hs2_kv_dtype dt, const float* lse, float* cand_score,
                                       int32_t* cand_idx, void* workspace,
                                       size_t workspace_bytes, hs2_stream_t stream);

/*
 * Step 5: from the G ranks' candidate lists in rank order (cand_score fp32,
 * cand_idx int32, both [G][B][T][topk]; the ranks' slices ascend), the global
 * selection of hs2_full_attn_select: the top-k by (score descending, position
 * ascending), then the window of query position q_pos0 + t, in idx int32
 * [B][T][topk + window] ascending (-1 padded) and n_sel int32 [B][T].
 * G * topk <= 51200.
 */
HS2_API hs2_status hs2_cp_merge_select(const float* cand_score, const int32_t* cand_idx, int G,
                                       int B, int T, int64_t q_pos0, int topk, int window,
                                       int32_t* idx, int32_t* n_sel, hs2_stream_t stream);

/*
 * hs2_sparse_attn -- a sparse-attention layer with KV Reuse (IT Home
 * announcement, "KV Reuse" paragraph: the sparse layers reuse the full
 * layer's KV cache and selection indices; the SWA branch is folded into the
 * forced window, so there is no second cache).
 *
 * For each query (b, t) and head h, over the positions S = idx[b][t][0 ..
 * n_sel[b][t]) of the same cache, softmax renormalised over S only:
 *   O[b][t][h][d] = sum_{j in S} softmax_j(scale * <Q[b][t][h], K[b][j]>) V[b][j][d]
 * Q is this layer's own bf16 [B][T][H][D]; idx/n_sel as written by
 * hs2_full_attn_select, with `slots` entries per query (>= n_sel).  Entries
 * outside [0, L) raise HS2_ERR_DEVICE through hs2_last_device_status and are
 * skipped.  A query with n_sel == 0 gets O = 0.
 * Supported: D in {64, 128}; H in {8, 16, 32}; slots <= 4096.
 * Ordering: the kernel is launched with programmatic dependent launch and
 * reads idx, n_sel and the K/V rows they name before waiting for the previous
 * kernel of the stream to finish (so that, in a block of sparse layers, it
 * gathers while the layer before it computes); after the wait it reads idx and
 * n_sel again and gathers anew if they changed.  Q is read after the wait.  A
 * kernel that precedes this call on the stream and itself lets dependent
 * launches start early must therefore not write the cache rows it uses after
 * doing so (this library's kernels never write the cache after letting a
 * dependent start).
 */
HS2_API hs2_status hs2_sparse_attn(const void* Q, const hs2_kv_cache* kv, int B, int T, int64_t L, int H,
                           int D, float scale, const int32_t* idx, const int32_t* n_sel,
                           int slots, hs2_kv_dtype dt, float* O, hs2_stream_t stream);

/*
 * hs2_full_attn_select_noalloc -- hs2_full_attn_select for callers that
 * cannot allocate device memory.  (The HySparse2 pages have no counterpart:
 * this is a packaging choice of this library.)
 *
 * Some callers have no way to obtain a workspace: code hosted by a framework
 * that reserves all device memory up front and hands its plugins no
 * allocator, or code on a latency-critical path that cannot afford
 * cudaMalloc's implicit device-wide synchronisation.  This entry point takes
 * the same arguments as hs2_full_attn_select minus the workspace, and uses a
 * scratch area built into the library instead: a static device array of
 * HS2_NOALLOC_SCRATCH_BYTES (16 MiB) that every GPU which loads libhs2 keeps
 * until the process exits.  It never calls cudaMalloc, cudaFree or any
 * allocating routine.
 *   - Arguments are checked exactly as hs2_full_attn_select checks them
 *     (HS2_ERR_INVALID_ARG / HS2_ERR_UNSUPPORTED) before the size: then a
 *     request whose workspace (hs2_full_attn_select_workspace) exceeds
 *     HS2_NOALLOC_SCRATCH_BYTES returns HS2_ERR_WORKSPACE.  Either way nothing
 *     is enqueued.  For example, 8 sequences of 32K positions need 4.6 MB.
 *   - The device address of the array is looked up (cudaGetSymbolAddress, on
 *     the caller's current device) by every call made outside stream capture;
 *     a call made while `stream` is being captured reuses the address found by
 *     the last call on that device outside capture, so make one call on each
 *     device before capturing it (the first call may also load the library's
 *     kernels, which capture forbids).  After a cudaDeviceReset, call once
 *     more outside capture before capturing again.
 *   - All calls on a device share the one array, and it keeps whatever the
 *     last call left there.  Every call clears on `stream` the parts that must
 *     start at zero: the fused kernel's arrival counters by a memset the call
 *     enqueues before the kernel, the selection histograms inside the kernels
 *     that fill them.  Calls whose work overlaps on the GPU (different
 *     streams, or different host threads) race on the array and must be
 *     serialised by the caller.
 * Outputs and status codes are those of hs2_full_attn_select.
 */
#define HS2_NOALLOC_SCRATCH_BYTES (16u << 20)
HS2_API hs2_status hs2_full_attn_select_noalloc(const void* Q, const hs2_kv_cache* kv, int B,
                                                int T, int64_t L, int H, int D, float scale,
                                                int topk, int window, hs2_kv_dtype dt, float* O,
                                                float* lse, int32_t* idx, int32_t* n_sel,
                                                hs2_stream_t stream);

/*
 * Waits for `stream`, then reads and clears the calling device's status
 * word: HS2_OK, HS2_ERR_TIMEOUT (a barrier wait gave up) or HS2_ERR_DEVICE
 * (an index was out of range).  HS2_ERR_CUDA if the wait itself failed.
 */
HS2_API hs2_status hs2_last_device_status(hs2_stream_t stream);

/* Static English description of a status code. */
HS2_API const char* hs2_status_string(hs2_status status);

/*
 * Optional timing of the dominant launch of hs2_full_attn_select (and of
 * hs2_full_attn_select_noalloc): the kernel that makes the one pass over the
 * whole K/V cache (for head_dim 128 and 32 query rows per group, the fused
 * kernel that also computes the scores and, when they fit, the selection).
 * While a pair is set, each of those calls made on this host thread records
 * `begin_event` on its stream just before that kernel and `end_event` just
 * after it, so that cudaEventElapsedTime of the pair is the kernel's device
 * time.  Inside stream capture the records become
 * external event nodes of the graph (cudaEventRecordExternal), recorded at
 * every replay.
 *   begin_event, end_event: cudaEvent_t handles owned by the caller, created
 *     with timing enabled; both null clears the pair (the default).
 * Returns HS2_ERR_INVALID_ARG when exactly one of the two is null.  Nothing is
 * enqueued by this call.
 */
HS2_API hs2_status hs2_set_stage_events(void* begin_event, void* end_event);

/*
 * Fault injection, for testing failure detection without a GPU fault.  While
 * extra_arrivals > 0, the group barriers of the fused full-attention kernel
 * (head_dim 128, 32 query rows per group, several CTAs per group) wait for
 * that many arrivals beyond the group's CTA count, which never come: every
 * such wait gives up after wait_limit_ns nanoseconds (0 = the default, one
 * second), raises HS2_ERR_TIMEOUT (read by hs2_last_device_status) and the
 * kernel's CTAs return with their outputs unfinished.  wait_limit_ns also
 * bounds those barriers when extra_arrivals is 0.  The setting applies to the
 * full-attention calls made afterwards on this host thread; (0, 0) restores
 * the defaults.  Nothing is enqueued by this call; it returns HS2_OK.
 */
HS2_API hs2_status hs2_set_fault_injection(unsigned extra_arrivals, unsigned long long wait_limit_ns);

/*
 * Phase timestamps of the fused full-attention kernel (the decode path of
 * hs2_full_attn_select: head_dim 128, 32 query rows per group), for tracing
 * where its time goes.  While `stamps` is set, every CTA b < max_ctas of that
 * kernel writes HS2_PHASES values of the GPU's nanosecond global timer to
 * stamps[b * HS2_PHASES + i]:
 *   0 CTA start, 1 its partial pass done (every K/V tile streamed and its
 *   partial written), 2 first group barrier passed, 3 its score pass done
 *   (candidate scores and histogram counts issued), 4 second group barrier
 *   passed, 5 third group barrier passed (selection), 6 CTA done; the eighth
 *   value is not written.
 * A stamp a CTA does not reach (a phase the call skips) is left as it was.
 *   stamps: device buffer of max_ctas * HS2_PHASES uint64 values, owned by the
 *     caller; NULL (the default) turns the stamps off.
 * The setting applies to the full-attention calls made afterwards on this host
 * thread.  Returns HS2_ERR_INVALID_ARG for a non-null stamps with max_ctas < 1
 * or a buffer not 8-byte aligned.  Nothing is enqueued by this call.
 */
#define HS2_PHASES 8
HS2_API hs2_status hs2_set_phase_stamps(unsigned long long* stamps, int max_ctas);

/* Library ABI version: 100 * major + minor. */
HS2_API int hs2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HS2_H */
