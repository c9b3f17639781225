// Internal launchers (C++ linkage, not part of the public ABI).  Shapes have
// been validated by the caller (hils_api.cu); these only enqueue kernels and
// return the launch error.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace hils {

struct Shape {
  int B, Hq, Hkv, G, N, d, S, W, nw, K, C, M;
  float scale;
  int dtype;  // 0 f32, 1 bf16
};

// K1: landmark summaries (all dtypes); shared_lmk: q_lmk is one query per head
// [Hq, d] shared by every chunk and sequence (the landmark-free variant)
cudaError_t launch_summaries(const Shape& s, const void* k, const void* q_lmk, void* k_sum, float* b_sum,
                             cudaStream_t st, const DevCtx& ctx, bool shared_lmk = false);

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
                                     int32_t* idx, float* s_sel, void* ws, cudaStream_t st, const DevCtx& ctx);

// fp32 SIMT prefill attention
cudaError_t launch_attn_prefill_simt(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                     const float* s_sel, void* out, cudaStream_t st, const DevCtx& ctx);

// bf16 prefill attention (d=128, S=64), one pass that streams each block's
// chunk union (no workspace)
cudaError_t launch_attn_prefill_tc(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                   const float* s_sel, void* out, cudaStream_t st, const DevCtx& ctx);
// the window pass over positions [t0, t1); with `part` (partial records of the
// selected chunks, tile of PT positions) it attends the window only and fuses
// the records, without it it also streams the selected chunks
cudaError_t launch_attn_window_merge(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                     const float* s_sel, void* out, const void* part, int t0, int t1, int PT,
                                     cudaStream_t st, const DevCtx& ctx);
// bf16 prefill attention, chunk-major selected chunks (tcgen05) + window pass,
// by position tiles; workspace of attn_prefill_tc_workspace(s) bytes
size_t attn_prefill_tc_workspace(const Shape& s);
cudaError_t launch_attn_prefill_chunked(const Shape& s, const void* q, const void* k, const void* v,
                                        const int32_t* idx, const float* s_sel, void* out, void* ws,
                                        cudaStream_t st, const DevCtx& ctx);

// decode attention (all dtypes): split-KV partials + merge
size_t decode_attn_workspace(const Shape& s);
cudaError_t launch_attn_decode(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                               const float* s_sel, void* out, void* ws, cudaStream_t st, const DevCtx& ctx);

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
