// Internal launchers (C++ linkage, not part of the public ABI).  Shapes have
// been validated by the caller (hils_api.cu); these only enqueue kernels and
// return the launch error.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "tmap.h"

namespace hils {

struct Shape {
  int B, Hq, Hkv, G, N, d, S, W, nw, K, C, M;
  float scale;
  int dtype;  // 0 f32, 1 bf16
};

// The decode cache as the decode kernels see it.  Default: every sequence has
// length N and its keys and values are contiguous [B, Hkv, N, d].  Paged: a
// pool of one-chunk pages [num_pages, Hkv, S, d]; chunk c of sequence b lives
// in page pages[b * max_pages + c]; sequence b has length seq_lens[b] <= N.
struct DecView {
  const int* seq_lens = nullptr;
  const int* pages = nullptr;
  int max_pages = 0;
  int num_pages = 0;
};
// cache length of sequence b
HILS_DI int dv_len(const DecView& v, const Shape& s, int b) { return v.seq_lens ? __ldg(v.seq_lens + b) : s.N; }
// element offset of the first key of chunk c of (sequence b, KV head g), or -1
// when the page table names a page outside the pool
HILS_DI long long dv_chunk(const DecView& v, const Shape& s, int b, int g, int c) {
  if (!v.pages) return (((long long)b * s.Hkv + g) * s.N + (long long)c * s.S) * s.d;
  if (c < 0 || c >= v.max_pages) return -1;
  const int p = __ldg(v.pages + (long long)b * v.max_pages + c);
  if (p < 0 || p >= v.num_pages) return -1;
  return ((long long)p * s.Hkv + g) * s.S * s.d;
}

// K1: landmark summaries (all dtypes); shared_lmk: q_lmk is one query per head
// [Hq, d] shared by every chunk and sequence (the landmark-free variant)
cudaError_t launch_summaries(const Shape& s, const void* k, const void* q_lmk, void* k_sum, float* b_sum,
                             cudaStream_t st, const DevCtx& ctx, bool shared_lmk = false);

// K1 on a paged decode cache (CUDA-core kernel): every complete chunk of each
// sequence (q_lmk [B, Hq, C, d]), or only the chunk the last token completed
// (last_only; q_lmk [B, Hq, d]); k_sum [B, Hq, C, d], b_sum [B, Hq, C]
cudaError_t launch_summaries_paged(const Shape& s, const void* k_pool, const void* q_lmk, void* k_sum, float* b_sum,
                                   const DecView& dv, bool last_only, cudaStream_t st, const DevCtx& ctx);
// the new token's key and value of each sequence into its page (position
// seq_lens[b] - 1); k_new, v_new [B, Hkv, d]
cudaError_t launch_decode_append(const Shape& s, const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                                 const DecView& dv, cudaStream_t st, const DevCtx& ctx);

// fp32 SIMT prefill score + group max + top-K
cudaError_t launch_score_topk_simt(const Shape& s, const void* q, const void* k_sum, const float* b_sum, int32_t* idx,
                                   float* s_sel, cudaStream_t st, const DevCtx& ctx);

// bf16 tensor-core prefill score + group max + top-K (d=128, S=64)
cudaError_t launch_score_topk_tc(const Shape& s, const void* q, const void* k_sum, const float* b_sum, int32_t* idx,
                                 float* s_sel, cudaStream_t st, const DevCtx& ctx);
size_t score_tc_workspace(const Shape& s);

// Q-Cal: q~ = q + W_up W_down h written to q_tilde [B,Hq,N,d] (bf16, d=128)
cudaError_t launch_qcal_tc(const Shape& s, const void* q, const void* h, const void* w_down, const void* w_up,
                           int rank, int d_model, void* q_tilde, cudaStream_t st, const DevCtx& ctx);

// decode score + group max + top-K (all dtypes); workspace: scores
size_t decode_score_workspace(const Shape& s);
cudaError_t launch_score_topk_decode(const Shape& s, const void* q, const void* k_sum, const float* b_sum,
                                     int32_t* idx, float* s_sel, void* ws, cudaStream_t st, const DevCtx& ctx,
                                     const DecView& dv = DecView{});

// fp32 SIMT prefill attention
cudaError_t launch_attn_prefill_simt(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                     const float* s_sel, void* out, cudaStream_t st, const DevCtx& ctx);

// bf16 prefill attention (d=128, S=64), one pass that streams each block's
// chunk union (no workspace)
cudaError_t launch_attn_prefill_tc(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                   const float* s_sel, void* out, cudaStream_t st, const DevCtx& ctx);
// window attention (tcgen05, two passes over the window chunks, attn_window.cu)
// of positions [t0, t0 + np) of a tile of PT positions (t0 a multiple of 32)
// into a window state of window_state_bytes(s, PT); then the fusion of that
// state with the partial records `part` of the selected chunks into out.  The
// tensor maps of q, k, v are made once per call.
struct WindowMaps {
  CUtensorMap q, k, v;
};
size_t window_state_bytes(const Shape& s, int PT);
cudaError_t make_window_maps(const Shape& s, const void* q, const void* k, const void* v, WindowMaps* m);
cudaError_t launch_attn_window(const Shape& s, const WindowMaps& m, void* wstate, int t0, int np, int PT,
                               cudaStream_t st, const DevCtx& ctx);
cudaError_t launch_attn_fuse(const Shape& s, const int32_t* idx, const float* s_sel, const void* part,
                             const void* wstate, void* out, int t0, int np, int PT, cudaStream_t st);
// bf16 prefill attention, chunk-major selected chunks (tcgen05) + window
// attention and fusion (attn_window.cu), by position tiles; workspace of
// attn_prefill_tc_workspace(s) bytes
size_t attn_prefill_tc_workspace(const Shape& s);
cudaError_t launch_attn_prefill_chunked(const Shape& s, const void* q, const void* k, const void* v,
                                        const int32_t* idx, const float* s_sel, void* out, void* ws,
                                        cudaStream_t st, const DevCtx& ctx);

// decode attention (all dtypes): split-KV partials + merge
size_t decode_attn_workspace(const Shape& s);
cudaError_t launch_attn_decode(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                               const float* s_sel, void* out, void* ws, cudaStream_t st, const DevCtx& ctx,
                               const DecView& dv = DecView{});

// decode attention with its partial records in a fixed device array (no allocation)
size_t decode_static_scratch_bytes();
cudaError_t launch_attn_decode_static(const Shape& s, const void* q, const void* k, const void* v,
                                      const int32_t* idx, const float* s_sel, void* out, cudaStream_t st,
                                      const DevCtx& ctx);

// backward of the prefill (attention, scores, summaries), CUDA-core kernels;
// workspace of prefill_bwd_workspace(s) bytes; ds_sel may be null
size_t prefill_bwd_workspace(const Shape& s);
cudaError_t launch_prefill_bwd(const Shape& s, const void* q, const void* k, const void* v, const void* q_lmk,
                               const int32_t* idx, const float* s_sel, const void* k_sum, const void* dout, float* dq,
                               float* dk, float* dv, float* dq_lmk, float* ds_sel, void* ws, cudaStream_t st,
                               const DevCtx& ctx);

}  // namespace hils
