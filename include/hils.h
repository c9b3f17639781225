/*
 * hils.h — C ABI of libhils.so: the forward hot path of Hierarchical Landmark
 * Sparse (HiLS) attention on NVIDIA B200 (sm_100a).
 *
 * Source of the method: the hyper.ai summary of arXiv 2607.02980
 * (HiLS-Attention), section "方法" (Method); cited below as [Method];
 * section "实验" (Experiments) of the same page is cited as [Exp].
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are DEVICE pointers to dense, row-major
 *    ("contiguous") buffers owned by the caller.  Element pointers must be
 *    16-byte aligned.  The library never allocates, frees or retains them.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call is asynchronous on that stream: it validates its
 *    arguments on the host, enqueues kernels and returns.
 *  - Notation: B batch, Hq query heads, Hkv key/value heads (G = Hq/Hkv
 *    query heads share one KV head, "a GQA group"), N sequence length,
 *    d head dim, S chunk size, C = floor(N/S) complete chunks, W window,
 *    n_w = W/S, K selected chunks, cur(i) = floor(i/S).
 *  - Window of position i: keys [max(0, (cur(i)-n_w+1)*S), i] (the current
 *    partial chunk plus the n_w-1 chunks before it).  Candidates of i: the
 *    complete chunks c <= cur(i)-n_w.  ([Method], uniform chunking and the
 *    chunk-aligned sliding window.)
 *  - dtype (hils_config_t.dtype) is the type of q, k, v, q_lmk, k_sum, out
 *    and of the Q-Cal tensors; scores (b_sum, s_sel) are always float32,
 *    chunk indices int32.
 *  - Errors: argument problems are caught on the host before any launch and
 *    return HILS_ERR_INVALID_ARG; shapes/dtypes without a kernel return
 *    HILS_ERR_UNSUPPORTED (there is no fallback of any kind); a failed launch
 *    returns HILS_ERR_CUDA.  A device-side wait that exceeds its budget sets
 *    a per-device status word and the kernel returns early; the caller sees it
 *    as HILS_ERR_TIMEOUT from hils_sync_status().  hils_last_error() gives a
 *    thread-local message for the last non-OK status.  No C++ exception
 *    crosses this boundary.
 *
 * Supported shapes (anything else returns HILS_ERR_UNSUPPORTED, checked on
 * the host before any launch):
 *  - every call: G in {1, 2, 4, 8}, K <= 64, n_w = W/S <= 32;
 *  - dtype F32 (CUDA-core kernels with fp32 FMA): d in {32, 64, 128} and
 *    S in {16, 32, 64}, except summaries with d = 32 and S = 64, prefill
 *    scoring with d = 128 and G = 8, and decode attention with d = 32 or
 *    S = 16;
 *  - dtype BF16 (tensor-core kernels): d = 128 and S = 64; prefill scoring
 *    and prefill attention need G = 4, and prefill attention N/S <= 8192;
 *    decode works for every G (its attention gathers tiles into warp-level
 *    MMAs); Q-Cal needs rank 64 and d_model a multiple of 64.
 */
#ifndef HILS_H
#define HILS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HILS_OK = 0,
  HILS_ERR_INVALID_ARG = 1,
  HILS_ERR_UNSUPPORTED = 2,
  HILS_ERR_CUDA = 3,
  HILS_ERR_TIMEOUT = 4
} hils_status_t;

typedef enum { HILS_F32 = 0, HILS_BF16 = 1 } hils_dtype_t;

typedef struct {
  int32_t batch;       /* B */
  int32_t seq_len;     /* N (prefill) or L, the decode cache length */
  int32_t n_q_heads;   /* Hq */
  int32_t n_kv_heads;  /* Hkv; Hq % Hkv == 0 */
  int32_t head_dim;    /* d */
  int32_t chunk;       /* S */
  int32_t window;      /* W; W % S == 0, W >= S */
  int32_t top_k;       /* K >= 1 */
  int32_t query_block; /* prefill tuning hint (0 = library default); never changes results */
  float scale;         /* logit scale; 0 means 1/sqrt(d) */
  int32_t dtype;       /* hils_dtype_t */
} hils_config_t;

/* Optional low-rank query calibration (Q-Cal), [Method] second practical
 * design choice: the scoring query is q~_i = q_i + W_up (W_down h_i), rank r.
 * It changes only the chunk scores, never the attention logits. */
typedef struct {
  const void* h;       /* [B, N, d_model] hidden states (dtype); decode: [B, d_model] */
  const void* w_down;  /* [r, d_model] (dtype) */
  const void* w_up;    /* [Hq*d, r] (dtype); row hq*d+e feeds head hq, dim e */
  int32_t rank;        /* r; the kernels support r = 64 */
  int32_t d_model;     /* a multiple of 64 */
} hils_qcal_t;

/*
 * Landmark chunk summaries, [Method] (paragraph after the surrogate-score
 * equation): for each (b, query head h, complete chunk c) the landmark query
 * q'_{h,c} induces p = softmax_j(q'_{h,c}.k_j * scale) over the S keys of
 * chunk c (KV head h/G); k'_{h,c} = sum_j p_j k_j and b'_{h,c} = the entropy
 * of p in nats.
 *   k      [B, Hkv, N, d]  (dtype)        q_lmk [B, Hq, C, d] (dtype)
 *   k_sum  [B, Hq, C, d]   (dtype, out)   b_sum [B, Hq, C]    (float32, out)
 * Decode uses the same call with N = L.
 */
hils_status_t hils_build_summaries(const hils_config_t* cfg, const void* k, const void* q_lmk, void* k_sum,
                                   float* b_sum, void* stream);

/*
 * The landmark-free variant of the summaries ([Method], last of the practical
 * design choices: one shared learnable query per layer takes the place of the
 * per-chunk landmark queries).  Read here as one query per query head,
 * shared by every chunk of every sequence: q'_{h,c} = q_shared[h] in the
 * computation of hils_build_summaries.
 *   k      [B, Hkv, N, d]  (dtype)        q_shared [Hq, d] (dtype)
 *   k_sum  [B, Hq, C, d]   (dtype, out)   b_sum    [B, Hq, C] (float32, out)
 * Shapes, errors and kernels are those of hils_build_summaries.
 */
hils_status_t hils_build_summaries_shared(const hils_config_t* cfg, const void* k, const void* q_shared,
                                          void* k_sum, float* b_sum, void* stream);

/*
 * Chunk scoring and top-K selection, [Method] surrogate-score equation and
 * third practical design choice (GQA):
 *   s^_{h,i,c} = q~_{h,i}.k'_{h,c} * scale + b'_{h,c}   for candidates c of i,
 *   g_{i,c}    = max over the G heads h of the group of s^_{h,i,c},
 *   I_i        = the K candidates with the largest g (ties: smaller c; all of
 *                them when there are fewer than K).
 * Outputs, per (b, KV group, position): idx = I_i in ascending chunk order,
 * padded with -1; per (b, query head, position): s_sel = that head's own s^ of
 * the chosen chunks, slot-aligned with idx, padded with -inf.
 *   prefill (decode = 0): q [B, Hq, N, d]; idx [B, Hkv, N, K]; s_sel [B, Hq, N, K]
 *   decode  (decode = 1): q [B, Hq, d] is the token at position L-1 (its key and
 *                         value are already in the cache); idx [B, Hkv, K];
 *                         s_sel [B, Hq, K]
 *   k_sum, b_sum: as produced by hils_build_summaries.
 *   qcal: NULL, or the Q-Cal tensors (prefill only).
 *   workspace: device scratch of at least
 *              hils_workspace_bytes(cfg, HILS_WS_SCORE_PREFILL or _DECODE, rank)
 *              bytes (may be NULL when that size is 0).  Contents on entry are
 *              ignored; the call owns it until the stream passes the call.
 */
hils_status_t hils_score_topk(const hils_config_t* cfg, const void* q, const hils_qcal_t* qcal, const void* k_sum,
                              const float* b_sum, int32_t* idx, float* s_sel, void* workspace, size_t ws_bytes,
                              int32_t decode, void* stream);

/*
 * Hierarchical-softmax sparse attention, prefill ([Method], the factorised
 * token weight w_{i,j} and the partition estimate Z^_i; the chatpaper abstract
 * of HiLS: each query attends every retrieved chunk on its own and the chunk
 * outputs are fused by the retrieval scores).  For query head h at position i:
 *   O_{i,c} = sum_{j in c} softmax_{j in c}(s_ij) v_j   (s_ij = q.k_j * scale)
 *   Z^_i    = sum_{c in I_i} exp(s^_c) + Z_swa,  Z_swa = sum_{j in window} exp(s_ij)
 *   out_i   = [sum_c exp(s^_c) O_{i,c} + sum_{j in window} exp(s_ij) v_j] / Z^_i
 * with s^_c taken from s_sel (each head its own).  Attention logits use the
 * raw q.
 *   q [B, Hq, N, d]; k, v [B, Hkv, N, d]; idx [B, Hkv, N, K]; s_sel [B, Hq, N, K];
 *   out [B, Hq, N, d] (dtype, out).
 * Each idx list must hold strictly ascending candidates of its position
 * followed by -1 padding (the form hils_score_topk writes).  Checked on the
 * device: an entry that is not a candidate, is not above every earlier entry
 * of its list, or follows a -1 is skipped (both attention passes skip the same
 * entries) and recorded in the status word, which hils_sync_status() reports
 * as HILS_ERR_INVALID_ARG.
 *   workspace: device scratch of at least
 *              hils_workspace_bytes(cfg, HILS_WS_ATTN_PREFILL, 0) bytes
 *              (16-byte aligned; 0 bytes for dtype F32; about 10 GB at
 *              B=1, N=128K, Hkv=8, K=32).  With it, bf16 runs attend the
 *              selected chunks chunk by chunk (the positions that chose a
 *              chunk share one load of its K and V tiles) and write one bf16
 *              partial record per (position, selected chunk) into the
 *              workspace, attend each position's window on the tensor cores,
 *              and fuse the two, by tiles of positions whose records fit about
 *              8 GiB.  Part of this work runs on an internal stream that waits
 *              on and is joined back into `stream` by events, so the call may
 *              be captured into a CUDA graph.  workspace = NULL with
 *              ws_bytes = 0 selects the pass that needs no scratch: each block
 *              of 14 positions streams the union of its chunks (slower on long
 *              contexts; same results within the bf16 tolerance).  The call
 *              owns the workspace until the stream passes it.
 */
hils_status_t hils_attn_prefill(const hils_config_t* cfg, const void* q, const void* k, const void* v,
                                const int32_t* idx, const float* s_sel, void* out, void* workspace,
                                size_t ws_bytes, void* stream);

/*
 * The same attention for one new token per sequence (decode), at position
 * L-1 of a cache of length L = cfg->seq_len.  The K chunks and the window are
 * split across CTAs and merged by a second kernel.
 *   q [B, Hq, d]; k_cache, v_cache [B, Hkv, L, d]; idx [B, Hkv, K];
 *   s_sel [B, Hq, K]; out [B, Hq, d] (dtype, out).
 *   idx lists have the form described at hils_attn_prefill and are checked
 *   the same way.
 *   workspace: at least hils_workspace_bytes(cfg, HILS_WS_ATTN_DECODE, 0)
 *              bytes of device scratch for the per-split partial results.
 */
hils_status_t hils_attn_decode(const hils_config_t* cfg, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* idx, const float* s_sel, void* out, void* workspace, size_t ws_bytes,
                               void* stream);

/*
 * hils_attn_decode without a workspace argument.  The paper has no
 * counterpart of this call: it exists for callers that cannot allocate
 * device memory for the call, e.g. a serving engine that has given all free
 * HBM to its own KV-cache pool, or a plug-in interface that hands over only
 * input and output buffers and has no allocator to offer.  Same arguments,
 * result and errors as hils_attn_decode, minus the workspace.
 *
 * The split-KV partial records go to one fixed device array inside the
 * library (4 MiB, i.e. B * Hq * nsplit * (d + 2) floats at most; nsplit is
 * the per-(sequence, group) split count, about 4 * SMs / (B * Hkv)).  Every
 * GPU that loads the library holds that array until the process exits.  A
 * configuration that needs more returns HILS_ERR_UNSUPPORTED with a message
 * naming both sizes; hils_workspace_bytes(cfg, HILS_WS_ATTN_DECODE, 0) gives
 * the need.  The call never allocates or frees memory.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  All calls share the one array and it keeps the last call's
 * contents: every record a call reads is written by the same call, so nothing
 * needs clearing, but two calls that overlap on the GPU (different streams,
 * or other threads) race on the array and must be serialised by the caller.
 */
hils_status_t hils_attn_decode_noalloc(const hils_config_t* cfg, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* idx, const float* s_sel, void* out,
                                       void* stream);

/*
 * Decode across steps on a paged, chunk-aligned KV cache, for sequences of
 * different lengths.  [Exp]: decode latency grows sublinearly with context
 * because a step touches only the token's K chunks and its window; so a cache
 * that grows by one token per step needs only the new token's key and value
 * written into place and, when that token completes a chunk, the summary of
 * that one chunk (no rebuild of the cache's summaries).
 *
 * The cache is a pool of one-chunk pages, k_pool / v_pool [num_pages, Hkv, S, d]
 * (dtype): chunk c of sequence b lives in page block_table[b * max_pages + c],
 * so one chunk of one KV head is one contiguous S x d tile.  cfg->seq_len is
 * the capacity L_max (it sets C = L_max / S, the chunk dimension of k_sum and
 * b_sum); sequence b has length seq_lens[b] in [1, L_max], its new token at
 * position seq_lens[b] - 1.  All arrays are device memory owned by the caller.
 * Checked on the device: a length outside [1, L_max] or a page outside
 * [0, num_pages) is skipped and reported (HILS_ERR_INVALID_ARG from
 * hils_sync_status()); never dereferenced.
 */
typedef struct {
  const int32_t* seq_lens;    /* [B] cache length of each sequence, new token included */
  const int32_t* block_table; /* [B, max_pages] pool page of chunk c of sequence b */
  int32_t max_pages;          /* >= ceil(cfg->seq_len / S) */
  int32_t num_pages;          /* pages in the pool */
} hils_paged_t;

/* Append one token per sequence: k_new, v_new [B, Hkv, d] go to position
 * seq_lens[b] - 1 of their pages (seq_lens already counts them).  If that
 * position ends a chunk (seq_lens[b] % S == 0), the chunk's summary is built
 * with its landmark query q_lmk_new[b] ([B, Hq, d]) into
 * k_sum [B, Hq, C, d] and b_sum [B, Hq, C] at chunk seq_lens[b] / S - 1
 * (the computation of hils_build_summaries for that chunk). */
hils_status_t hils_decode_append(const hils_config_t* cfg, const hils_paged_t* paged, const void* k_new,
                                 const void* v_new, const void* q_lmk_new, void* k_pool, void* v_pool, void* k_sum,
                                 float* b_sum, void* stream);

/* Summaries of every complete chunk of each sequence of a paged cache
 * (q_lmk [B, Hq, C, d]; chunks past a sequence's length are left untouched),
 * e.g. after a prefill written into the pool. */
hils_status_t hils_build_summaries_paged(const hils_config_t* cfg, const hils_paged_t* paged, const void* k_pool,
                                         const void* q_lmk, void* k_sum, float* b_sum, void* stream);

/* hils_score_topk (decode = 1) for sequences of the given lengths: the
 * candidates of sequence b are its complete chunks before the window of
 * position seq_lens[b] - 1.  Workspace: HILS_WS_SCORE_DECODE. */
hils_status_t hils_score_topk_paged(const hils_config_t* cfg, const void* q, const hils_paged_t* paged,
                                    const void* k_sum, const float* b_sum, int32_t* idx, float* s_sel,
                                    void* workspace, size_t ws_bytes, void* stream);

/* hils_attn_decode on the paged cache, each sequence at its own length.
 * Workspace: HILS_WS_ATTN_DECODE. */
hils_status_t hils_attn_decode_paged(const hils_config_t* cfg, const void* q, const void* k_pool, const void* v_pool,
                                     const hils_paged_t* paged, const int32_t* idx, const float* s_sel, void* out,
                                     void* workspace, size_t ws_bytes, void* stream);

/*
 * Device address of page-locked (pinned), mapped host memory, for keeping the
 * decode KV cache in host memory (the wmrh.cn article on HiLS: chunk-sparse
 * attention lets the unselected chunks of the cache stay off the GPU).  Passed
 * as k_cache / v_cache to hils_attn_decode (or as the pools of
 * hils_attn_decode_paged), the decode attention reads only the token's K
 * chunks and its window, i.e. (K S + W) Hkv d 2 elements per sequence, over
 * the host link; the summaries stay in device memory.  Returns
 * HILS_ERR_INVALID_ARG (and launches nothing) if `host` is not such memory.
 */
hils_status_t hils_host_device_pointer(const void* host, void** device_ptr);

/*
 * The whole prefill path from host memory: copies the inputs to the device,
 * builds the summaries, scores and selects (hils_build_summaries,
 * hils_score_topk) and attends (hils_attn_prefill), then copies the output
 * back.  The pages have no counterpart of this call; it packages the three
 * steps above with their transfers so that a caller holding the inputs in
 * host memory gets the output in host memory.
 *
 * Every (sequence, KV group) is an independent piece of the computation (its
 * G query heads, its keys and values, its chunk lists).  Without Q-Cal the
 * call uploads, computes and downloads piece by piece on two internal copy
 * streams, so that the transfers of one piece overlap the kernels of others;
 * with Q-Cal (whose low-rank term is shared by all heads) it uploads all
 * inputs, scores the whole problem, then attends and downloads by piece.
 * The results are those of the three device calls.
 *   h_q [B, Hq, N, d], h_k / h_v [B, Hkv, N, d], h_q_lmk [B, Hq, C, d]
 *   (dtype, host); h_out [B, Hq, N, d] (dtype, host, written).
 *   qcal: NULL, or the Q-Cal tensors in HOST memory (layouts of hils_qcal_t).
 *   Host buffers should be page-locked (cudaHostAlloc / pinned); pageable
 *   memory works but the copies then do not overlap the kernels.
 *   workspace: device memory of at least
 *              hils_workspace_bytes(cfg, HILS_WS_PREFILL_HOST, rank) bytes
 *              (16-byte aligned); it holds the device copies of the inputs and
 *              all intermediate tensors, and belongs to the call until
 *              `stream` passes it.
 * The call enqueues all work and returns: h_out is complete once `stream`
 * has passed the call (hils_sync_status(stream) waits and reports device
 * errors).  The host buffers must stay valid and unchanged until then.  The
 * call waits on and records events of its internal streams, so it must not be
 * captured into a CUDA graph.
 */
hils_status_t hils_prefill_host(const hils_config_t* cfg, const void* h_q, const void* h_k, const void* h_v,
                                const void* h_q_lmk, const hils_qcal_t* qcal, void* h_out, void* workspace,
                                size_t ws_bytes, void* stream);

/*
 * Backward of the prefill: gradients of a loss L with respect to q, k, v and
 * the landmark queries, given dL/dout, with the chunk selection idx held fixed
 * (top-K is a discrete choice).  [Method], the factorised token weight w_ij
 * and Z^_i: the loss reaches each chosen chunk's score s^ through its fusion
 * weight exp(s^)/Z^, and from s^ = q.k'/sqrt(d) + b' the landmark summaries
 * k', b' and their queries q'_c (the wmrh.cn article on HiLS: the hierarchical
 * softmax lets the language-model loss train the summaries).  The scoring
 * query is q (no Q-Cal).
 *   q [B,Hq,N,d], k, v [B,Hkv,N,d], q_lmk [B,Hq,C,d], k_sum [B,Hq,C,d] (dtype):
 *     the forward's inputs and its summaries;
 *   idx [B,Hkv,N,K], s_sel [B,Hq,N,K]: the forward's selection and scores
 *     (lists in the form of hils_attn_prefill, checked the same way);
 *   dout [B,Hq,N,d] (dtype): dL/dout.
 * Outputs, float32, overwritten: dq [B,Hq,N,d] (attention logits and score
 * path), dk, dv [B,Hkv,N,d] (attention, and for dk the summaries),
 * dq_lmk [B,Hq,C,d]; ds_sel [B,Hq,N,K] = dL/ds^ per chosen slot (0 elsewhere),
 * or NULL.  Kernels: CUDA cores, fp32 arithmetic, no floating-point atomics
 * on global memory.  dq and ds_sel repeat bit for bit; dk, dv and dq_lmk sum
 * a chunk's rows in the order of its bucket list (filled by atomic arrival),
 * so repeats agree to fp32 rounding.  workspace: at least
 * hils_workspace_bytes(cfg, HILS_WS_PREFILL_BWD, 0) bytes.  Shapes: those of
 * the forward's summaries and attention for the dtype (fp32: d in
 * {32, 64, 128}; bf16: d = 128, S = 64), any G.
 */
hils_status_t hils_prefill_bwd(const hils_config_t* cfg, const void* q, const void* k, const void* v,
                               const void* q_lmk, const int32_t* idx, const float* s_sel, const void* k_sum,
                               const void* dout, float* dq, float* dk, float* dv, float* dq_lmk, float* ds_sel,
                               void* workspace, size_t ws_bytes, void* stream);

enum {
  HILS_WS_SCORE_PREFILL = 0,
  HILS_WS_SCORE_DECODE = 1,
  HILS_WS_ATTN_DECODE = 2,
  HILS_WS_PREFILL_HOST = 3,
  HILS_WS_ATTN_PREFILL = 4,
  HILS_WS_PREFILL_BWD = 5
};

/* Bytes of workspace the call `which` needs for this configuration (0 if none);
 * qcal_rank is the Q-Cal rank for HILS_WS_SCORE_PREFILL and
 * HILS_WS_PREFILL_HOST (0 = no Q-Cal).  With Q-Cal, hils_prefill_host
 * supports d_model = Hq * d only (so that this size is known from cfg) and
 * returns HILS_ERR_UNSUPPORTED for any other width.
 * Returns (size_t)-1 for an invalid configuration. */
size_t hils_workspace_bytes(const hils_config_t* cfg, int32_t which, int32_t qcal_rank);

/* Synchronises `stream`, then reads and clears the calling device's status
 * word: HILS_OK, HILS_ERR_TIMEOUT (a bounded device wait ran out), or
 * HILS_ERR_INVALID_ARG (a kernel skipped a chunk-list entry that was not a
 * candidate, not ascending, or after the list's -1 padding). */
hils_status_t hils_sync_status(void* stream);

/* Thread-local text for the last non-OK status returned on this thread. */
const char* hils_last_error(void);

/* Test hook: budget, in clock64 cycles, of every bounded device wait launched
 * after this call (0 restores the default of about 2 s at 2 GHz). */
void hils_set_wait_budget(int64_t cycles);

/* Test hook: mode 1 makes every kernel launched afterwards that waits on
 * tile copies (decode attention, tensor-core prefill) skip issuing those
 * copies, so that its bounded waits run out with no copy left in flight; the
 * kernels then return early and hils_sync_status() reports HILS_ERR_TIMEOUT.
 * Outputs of such launches are undefined.  mode 0 turns the hook off. */
void hils_set_fault_injection(int32_t mode);

/* Library version, e.g. "hils-b200 1.0". */
const char* hils_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HILS_H */
