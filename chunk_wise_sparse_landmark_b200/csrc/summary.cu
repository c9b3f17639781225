// K1 — landmark chunk summaries.
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method), the paragraph after the surrogate-score equation: the landmark
// query q'_c of a chunk induces an attention distribution p over the chunk's
// keys; k'_c is the p-weighted sum of those keys and b'_c the entropy of p.
//
// One CTA (256 threads) handles one (batch, KV head, chunk) at a time and
// serves all G query heads of the group, so each key tile is read from HBM
// once.  The tile is staged in shared memory as fp32 with a padded row pitch
// (conflict-free column and row walks); logits, the softmax and the entropy
// are fp32.  The entropy is evaluated as (m + log Z) - sum p*l, which avoids
// 0*log 0.  The kernel is HBM-bound: it reads K once and writes G summaries.
#include "gather_mma.cuh"
#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int kThreads = 256;

// Element offset of the landmark query of (sequence b, query head h, chunk c):
// per-chunk queries use strides (Hq C d, C d, d); the landmark-free variant's
// one shared query per head uses (0, d, 0).
struct LmkStrides {
  long long b, h, c;
  HILS_DI long long of(int bb, int hh, int cc) const { return bb * b + hh * h + cc * c; }
};

// Which chunks a launch summarises.  kAllChunks: every complete chunk of a
// contiguous cache [B, Hkv, N, d].  kPagedAll: every complete chunk of each
// sequence of a paged cache (units over max_pages, those past the sequence's
// length skipped).  kPagedLast: the chunk that the last token of each sequence
// completed, if it completed one (length % S == 0), with its landmark query
// given per sequence (chunk stride 0 in LmkStrides).
enum SummUnits { kAllChunks = 0, kPagedAll = 1, kPagedLast = 2 };

template <typename T, int D, int S, int G>
__global__ void __launch_bounds__(kThreads) summaries_kernel(Shape s, const T* __restrict__ k,
                                                             const T* __restrict__ q_lmk, LmkStrides ls,
                                                             T* __restrict__ k_sum, float* __restrict__ b_sum,
                                                             DecView dv, int mode, DevCtx ctx) {
  __shared__ float ks[S][D + 1];
  __shared__ float qs[G][D];
  __shared__ float lg[G][S];
  const int tid = threadIdx.x;
  const int per = mode == kAllChunks ? s.C : mode == kPagedAll ? dv.max_pages : 1;
  const long long units = (long long)s.B * s.Hkv * per;
  for (long long u = blockIdx.x; u < units; u += gridDim.x) {
    int c = (int)(u % per);
    const int g = (int)((u / per) % s.Hkv);
    const int b = (int)(u / ((long long)per * s.Hkv));
    long long koff;
    if (mode == kAllChunks) {
      koff = (((long long)b * s.Hkv + g) * s.N + (long long)c * S) * D;
    } else {
      const int L = dv_len(dv, s, b);
      if (L < 1 || L > s.N) {
        if (tid == 0 && g == 0 && c == 0) raise_status(ctx, kStatusBadIndex);
        continue;
      }
      if (mode == kPagedLast) {
        if (L % S) continue;  // the last token completed no chunk
        c = L / S - 1;
      } else if (c >= L / S) {
        continue;  // not a complete chunk of this sequence
      }
      koff = dv_chunk(dv, s, b, g, c);
      if (koff < 0) {  // a page outside the pool: reported, never read
        if (tid == 0) raise_status(ctx, kStatusBadIndex);
        continue;
      }
    }
    const T* kc = k + koff;
    for (int e = tid; e < S * D; e += kThreads) ks[e / D][e % D] = to_f32(kc[e]);
    for (int e = tid; e < G * D; e += kThreads) {
      const int hg = e / D;
      qs[hg][e % D] = to_f32(q_lmk[ls.of(b, g * G + hg, c) + e % D]);
    }
    __syncthreads();
    // logits l[h][j] = q'_h . k_j * scale
    for (int p = tid; p < G * S; p += kThreads) {
      const int hg = p / S, j = p % S;
      float acc = 0.f;
#pragma unroll 8
      for (int e = 0; e < D; ++e) acc = fmaf(qs[hg][e], ks[j][e], acc);
      lg[hg][j] = acc * s.scale;
    }
    __syncthreads();
    // per head: softmax over the S keys, entropy
    const int warp = tid >> 5, lane = tid & 31;
    for (int hg = warp; hg < G; hg += kThreads / 32) {
      float m = -INFINITY;
      for (int j = lane; j < S; j += 32) m = fmaxf(m, lg[hg][j]);
      m = warp_max(m);
      float z = 0.f, zl = 0.f;
      for (int j = lane; j < S; j += 32) {
        const float e = expf(lg[hg][j] - m);
        z += e;
        zl += e * lg[hg][j];
      }
      z = warp_sum(z);
      zl = warp_sum(zl);
      __syncwarp();
      for (int j = lane; j < S; j += 32) lg[hg][j] = expf(lg[hg][j] - m) / z;
      if (lane == 0) b_sum[((long long)b * s.Hq + g * G + hg) * s.C + c] = (m + logf(z)) - zl / z;
    }
    __syncthreads();
    // k'_h = sum_j p_hj k_j
    for (int o = tid; o < G * D; o += kThreads) {
      const int hg = o / D, e = o % D;
      float acc = 0.f;
#pragma unroll 8
      for (int j = 0; j < S; ++j) acc = fmaf(lg[hg][j], ks[j][e], acc);
      k_sum[(((long long)b * s.Hq + g * G + hg) * s.C + c) * D + e] = from_f32<T>(acc);
    }
    __syncthreads();
  }
}

template <typename T, int D, int S, int G>
cudaError_t go(const Shape& s, const void* k, const void* q_lmk, const LmkStrides& ls, void* k_sum, float* b_sum,
               cudaStream_t st, const DevCtx& ctx, const DecView& dv = DecView{}, int mode = kAllChunks) {
  const int per = mode == kAllChunks ? s.C : mode == kPagedAll ? dv.max_pages : 1;
  const long long units = (long long)s.B * s.Hkv * per;
  if (units == 0) return cudaSuccess;
  const int sms = device_sm_count();
  const long long grid = units < (long long)sms * 8 ? units : (long long)sms * 8;
  summaries_kernel<T, D, S, G><<<(unsigned)grid, kThreads, 0, st>>>(s, (const T*)k, (const T*)q_lmk, ls, (T*)k_sum,
                                                                     b_sum, dv, mode, ctx);
  return cudaGetLastError();
}

template <typename T, int D, int S>
cudaError_t go_g(const Shape& s, const void* k, const void* q_lmk, const LmkStrides& ls, void* k_sum, float* b_sum,
                 cudaStream_t st, const DevCtx& ctx, const DecView& dv, int mode) {
  switch (s.G) {
    case 1: return go<T, D, S, 1>(s, k, q_lmk, ls, k_sum, b_sum, st, ctx, dv, mode);
    case 2: return go<T, D, S, 2>(s, k, q_lmk, ls, k_sum, b_sum, st, ctx, dv, mode);
    case 4: return go<T, D, S, 4>(s, k, q_lmk, ls, k_sum, b_sum, st, ctx, dv, mode);
    case 8: return go<T, D, S, 8>(s, k, q_lmk, ls, k_sum, b_sum, st, ctx, dv, mode);
  }
  return cudaErrorNotSupported;
}

template <typename T>
cudaError_t go_t(const Shape& s, const void* k, const void* q_lmk, const LmkStrides& ls, void* k_sum, float* b_sum,
                 cudaStream_t st, const DevCtx& ctx, const DecView& dv = DecView{}, int mode = kAllChunks) {
#define HILS_CASE(DD, SS) \
  if (s.d == DD && s.S == SS) return go_g<T, DD, SS>(s, k, q_lmk, ls, k_sum, b_sum, st, ctx, dv, mode);
  HILS_CASE(64, 32)
  HILS_CASE(64, 64)
  HILS_CASE(128, 32)
  HILS_CASE(128, 64)
  HILS_CASE(32, 16)
  HILS_CASE(64, 16)
  HILS_CASE(128, 16)
  HILS_CASE(32, 32)
#undef HILS_CASE
  return cudaErrorNotSupported;
}

// ---------------------------------------------------------------------------
// bf16, d = 128, S = 64: one warp per (batch, KV head, chunk) at a time.  The
// summary is a small attention with the keys as values:
//   S^T (64 keys x 8 cols) = K_c . Q'^T,  p = softmax over keys per column,
//   k'^T (128 x 8 cols)    = K_c^T . P^T
// on the tensor cores (bf16 mma.sync, fp32 accumulation), with the group's
// G <= 8 landmark queries as the N = 8 columns.  P is split into bf16 hi + lo
// parts (two MMAs) so k' keeps close to fp32 accuracy before its final bf16
// rounding; the entropy uses the fp32 logits.  Fragment layouts and
// line-wide loads: gather_mma.cuh; the second read of the tile hits L1.
template <int G>
__global__ void __launch_bounds__(256) summaries_mma(Shape s, const __nv_bfloat16* __restrict__ k,
                                                     const __nv_bfloat16* __restrict__ q_lmk, LmkStrides ls,
                                                     __nv_bfloat16* __restrict__ k_sum, float* __restrict__ b_sum) {
  constexpr int D = 128, S = 64;
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2, c4 = lane & 3;
  const long long units = (long long)s.B * s.Hkv * s.C;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long u = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < units; u += warps) {
    const int c = (int)(u % s.C);
    const int g = (int)((u / s.C) % s.Hkv);
    const int b = (int)(u / ((long long)s.C * s.Hkv));
    const __nv_bfloat16* kc = k + (((long long)b * s.Hkv + g) * s.N + (long long)c * S) * D;
    // Q'^T as the B operand: column gq = landmark query of head g*G + gq
    uint32_t qf[2][8];
    load_qcol(gq < G ? q_lmk + ls.of(b, g * G + gq, c) : nullptr, c4, qf);
    float sc[4][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
    mma_st_tile(kc, S - 1, gq, c4, qf, sc);
    // softmax per column, entropy = (m + log Z) - sum p l
    float phi[4][4], plo[4][4];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        sc[mt][r] *= s.scale;
        sc[mt][2 + r] *= s.scale;
        mx = fmaxf(mx, fmaxf(sc[mt][r], sc[mt][2 + r]));
      }
      mx = col_max(mx);
      float z = 0.f, zl = 0.f;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const float l = sc[mt][2 * hi + r];
          const float e = expf(l - mx);
          sc[mt][2 * hi + r] = e;
          z += e;
          zl += e * l;
        }
      z = col_sum(z);
      zl = col_sum(zl);
      const float inv = 1.f / z;
      const int hcol = 2 * c4 + r;
      if (hcol < G && gq == 0) b_sum[((long long)b * s.Hq + g * G + hcol) * s.C + c] = (mx + logf(z)) - zl * inv;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const float p = sc[mt][2 * hi + r] * inv;
          const float ph = __bfloat162float(__float2bfloat16_rn(p));
          phi[mt][2 * hi + r] = ph;
          plo[mt][2 * hi + r] = p - ph;
        }
    }
    // k'^T = K^T P^T (hi and lo parts)
    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    mma_ot_tile(kc, S - 1, gq, c4, phi, acc);
    mma_ot_tile(kc, S - 1, gq, c4, plo, acc);
    // thread holds dims 8 gq + mt (acc[mt][r]) and 64 + 8 gq + mt (acc[mt][2 + r]) of columns 2c4 + r
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int hcol = 2 * c4 + r;
      if (hcol >= G) continue;
      __nv_bfloat16* o = k_sum + (((long long)b * s.Hq + g * G + hcol) * s.C + c) * D;
      uint4 lo, hi;
      lo.x = pack_bf16x2(acc[0][r], acc[1][r]);
      lo.y = pack_bf16x2(acc[2][r], acc[3][r]);
      lo.z = pack_bf16x2(acc[4][r], acc[5][r]);
      lo.w = pack_bf16x2(acc[6][r], acc[7][r]);
      hi.x = pack_bf16x2(acc[0][2 + r], acc[1][2 + r]);
      hi.y = pack_bf16x2(acc[2][2 + r], acc[3][2 + r]);
      hi.z = pack_bf16x2(acc[4][2 + r], acc[5][2 + r]);
      hi.w = pack_bf16x2(acc[6][2 + r], acc[7][2 + r]);
      *reinterpret_cast<uint4*>(o + 8 * gq) = lo;
      *reinterpret_cast<uint4*>(o + 64 + 8 * gq) = hi;
    }
  }
}

template <int G>
cudaError_t go_mma(const Shape& s, const void* k, const void* q_lmk, const LmkStrides& ls, void* k_sum, float* b_sum,
                   cudaStream_t st) {
  const long long units = (long long)s.B * s.Hkv * s.C;
  if (units == 0) return cudaSuccess;
  const long long blocks_needed = (units + 7) / 8;
  const long long cap = (long long)device_sm_count() * 8;
  const unsigned grid = (unsigned)(blocks_needed < cap ? blocks_needed : cap);
  summaries_mma<G><<<grid, 256, 0, st>>>(s, (const __nv_bfloat16*)k, (const __nv_bfloat16*)q_lmk, ls,
                                         (__nv_bfloat16*)k_sum, b_sum);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_summaries(const Shape& s, const void* k, const void* q_lmk, void* k_sum, float* b_sum,
                             cudaStream_t st, const DevCtx& ctx, bool shared_lmk) {
  // per-chunk landmark queries [B, Hq, C, d], or one shared query per head [Hq, d]
  const LmkStrides ls = shared_lmk ? LmkStrides{0, (long long)s.d, 0}
                                   : LmkStrides{(long long)s.Hq * s.C * s.d, (long long)s.C * s.d, (long long)s.d};
  if (s.dtype == 0) return go_t<float>(s, k, q_lmk, ls, k_sum, b_sum, st, ctx);
  if (s.d == 128 && s.S == 64) {
    switch (s.G) {
      case 1: return go_mma<1>(s, k, q_lmk, ls, k_sum, b_sum, st);
      case 2: return go_mma<2>(s, k, q_lmk, ls, k_sum, b_sum, st);
      case 4: return go_mma<4>(s, k, q_lmk, ls, k_sum, b_sum, st);
      case 8: return go_mma<8>(s, k, q_lmk, ls, k_sum, b_sum, st);
    }
  }
  return go_t<__nv_bfloat16>(s, k, q_lmk, ls, k_sum, b_sum, st, ctx);
}

cudaError_t launch_summaries_paged(const Shape& s, const void* k_pool, const void* q_lmk, void* k_sum, float* b_sum,
                                   const DecView& dv, bool last_only, cudaStream_t st, const DevCtx& ctx) {
  // every chunk: q_lmk [B, Hq, C, d]; the chunk the last token completed: q_lmk [B, Hq, d]
  const LmkStrides ls = last_only ? LmkStrides{(long long)s.Hq * s.d, (long long)s.d, 0}
                                  : LmkStrides{(long long)s.Hq * s.C * s.d, (long long)s.C * s.d, (long long)s.d};
  const int mode = last_only ? kPagedLast : kPagedAll;
  if (s.dtype == 0) return go_t<float>(s, k_pool, q_lmk, ls, k_sum, b_sum, st, ctx, dv, mode);
  return go_t<__nv_bfloat16>(s, k_pool, q_lmk, ls, k_sum, b_sum, st, ctx, dv, mode);
}

}  // namespace hils
