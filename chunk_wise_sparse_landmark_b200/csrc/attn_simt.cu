// Hierarchical-softmax sparse attention, fp32 prefill path (CUDA cores).
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method): the token weight w_{i,j} = exp(s_ij)/Z_{i,c(j)} * exp(s^_{i,c(j)})/Z^_i
// with Z^_i = sum_{c in I_i} exp(s^_{i,c}) + Z_{i,swa}; chatpaper abstract of
// HiLS: each query attends each retrieved chunk on its own and the chunk
// outputs are fused by the retrieval scores.
//
// One warp per (batch, query head, position); lanes split the head
// dimension.  Each unit (the window, or one selected chunk) is reduced with
// its own online softmax and then folded into the fused output with log-space
// weight A (A = s^ of the chunk, or LSE of the window logits), all shifted by
// the running maximum of A.  True FP32 FMA throughout.
#include "launch.h"

namespace hils {
namespace {

template <int D>
__global__ void __launch_bounds__(256) attn_prefill_simt(Shape s, const float* __restrict__ q,
                                                          const float* __restrict__ k, const float* __restrict__ v,
                                                          const int32_t* __restrict__ idx,
                                                          const float* __restrict__ s_sel, float* __restrict__ out,
                                                          DevCtx ctx) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long rows = (long long)s.B * s.Hq * s.N;
  if (row >= rows) return;
  const int i = (int)(row % s.N);
  const int h = (int)((row / s.N) % s.Hq);
  const int b = (int)(row / ((long long)s.N * s.Hq));
  const int g = h / s.G;
  const float* qi = q + row * D;
  const float* kb = k + ((long long)b * s.Hkv + g) * (long long)s.N * D;
  const float* vb = v + ((long long)b * s.Hkv + g) * (long long)s.N * D;
  float qr[E];
#pragma unroll
  for (int e = 0; e < E; ++e) qr[e] = qi[lane + 32 * e];

  // fused accumulator: num = sum e^{A - Mf} O_unit, den = sum e^{A - Mf}
  float Mf = -INFINITY, den = 0.f, num[E];
#pragma unroll
  for (int e = 0; e < E; ++e) num[e] = 0.f;

  auto unit = [&](int j0, int j1, bool selected, float a_sel) {
    float m = -INFINITY, l = 0.f, o[E];
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = 0.f;
    for (int j = j0; j <= j1; ++j) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) acc = fmaf(qr[e], kb[(long long)j * D + lane + 32 * e], acc);
      const float sj = warp_sum(acc) * s.scale;
      const float mn = fmaxf(m, sj);
      const float corr = expf(m - mn), p = expf(sj - mn);
      l = l * corr + p;
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = o[e] * corr + p * vb[(long long)j * D + lane + 32 * e];
      m = mn;
    }
    // unit contributes e^{A} * (o / l):  A = s^ (selected) or m + log l (window)
    const float A = selected ? a_sel : m + logf(l);
    const float Mn = fmaxf(Mf, A);
    const float cf = expf(Mf - Mn), cu = expf(A - Mn);
    den = den * cf + cu;
#pragma unroll
    for (int e = 0; e < E; ++e) num[e] = num[e] * cf + cu * (o[e] / l);
    Mf = Mn;
  };

  // window: keys [max(0, (cur - nw + 1) S), i]
  const int cur = i / s.S;
  const int ws = max(0, (cur - s.nw + 1) * s.S);
  unit(ws, i, false, 0.f);
  // selected chunks
  const int ncand = max(0, cur - s.nw + 1);
  const int32_t* ir = idx + (((long long)b * s.Hkv + g) * s.N + i) * s.K;
  const float* sr = s_sel + row * s.K;
  // the list form (common.cuh, accept_list_warp): ascending candidates, then -1
  int prev = -1;  // largest entry so far; a negative entry ends the list
  for (int x = 0; x < s.K; ++x) {
    const int c = ir[x];
    const bool ok = c >= 0 && c < ncand && c > prev;
    if (!ok) {
      if (c != -1 && lane == 0) raise_status(ctx, kStatusBadIndex);
      prev = c < 0 ? 0x7fffffff : max(prev, c);
      continue;
    }
    prev = c;
    unit(c * s.S, c * s.S + s.S - 1, true, sr[x]);
  }
  float* o = out + row * D;
#pragma unroll
  for (int e = 0; e < E; ++e) o[lane + 32 * e] = num[e] / den;
}

}  // namespace

cudaError_t launch_attn_prefill_simt(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                     const float* s_sel, void* out, cudaStream_t st, const DevCtx& ctx) {
  const long long rows = (long long)s.B * s.Hq * s.N;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  switch (s.d) {
    case 32:
      attn_prefill_simt<32><<<grid, 256, 0, st>>>(s, (const float*)q, (const float*)k, (const float*)v, idx, s_sel,
                                                   (float*)out, ctx);
      break;
    case 64:
      attn_prefill_simt<64><<<grid, 256, 0, st>>>(s, (const float*)q, (const float*)k, (const float*)v, idx, s_sel,
                                                   (float*)out, ctx);
      break;
    case 128:
      attn_prefill_simt<128><<<grid, 256, 0, st>>>(s, (const float*)q, (const float*)k, (const float*)v, idx, s_sel,
                                                    (float*)out, ctx);
      break;
    default:
      return cudaErrorNotSupported;
  }
  return cudaGetLastError();
}

}  // namespace hils
