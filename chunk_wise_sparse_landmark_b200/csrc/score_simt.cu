// Chunk scoring, GQA group max and top-K on CUDA cores.
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method): the surrogate score s^_{i,c} = q_i.k'_c / sqrt(d) + b'_c, chunks
// ranked by s^ and the top K kept; third practical design choice: scores are
// computed per head, reduced by a max over the heads of each GQA group, and
// the top K chunks are chosen from the group score.  Only complete chunks
// that lie before the chunk-aligned window are candidates.
//
// Two kernels live here:
//  * score_topk_prefill_simt — the fp32 prefill path (true FP32 FMA, which
//    the fp32 tolerance needs).  One thread per (position, head) keeps its
//    query in registers; per-position top-K lists live in shared memory.
//  * the decode path (one query per sequence, every dtype): a bandwidth-bound
//    pass that streams k' once and writes per-head and group scores to the
//    workspace, then a per-(sequence, group) radix select that picks the K
//    best chunks deterministically (ties: smaller chunk index).
#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

// ------------------------------------------------------------ prefill fp32 --
constexpr int kQB = 32;  // positions per CTA
constexpr int kTC = 8;   // chunks per shared-memory tile

template <int D, int G, int KMAX>
__global__ void __launch_bounds__(kQB* G) score_topk_prefill_simt(Shape s, const float* __restrict__ q,
                                                                   const float* __restrict__ k_sum,
                                                                   const float* __restrict__ b_sum,
                                                                   int32_t* __restrict__ idx,
                                                                   float* __restrict__ s_sel) {
  __shared__ float kt[G][kTC][D];
  __shared__ float bt[G][kTC];
  __shared__ float st[kQB][G][kTC + 1];
  __shared__ float lg[kQB][KMAX];
  __shared__ int lc[kQB][KMAX];
  const int tid = threadIdx.x;
  const int qi = tid / G, hg = tid % G;
  const int g = blockIdx.y, b = blockIdx.z;
  const int i0 = blockIdx.x * kQB;
  const int i = i0 + qi;
  const int h = g * G + hg;
  const bool valid = i < s.N;
  float qr[D];
#pragma unroll
  for (int e = 0; e < D; ++e) qr[e] = valid ? q[(((long long)b * s.Hq + h) * s.N + i) * D + e] : 0.f;
  const int ncand = valid ? max(0, i / s.S - s.nw + 1) : 0;
  const int last_i = min(i0 + kQB, s.N) - 1;
  const int ncand_blk = max(0, last_i / s.S - s.nw + 1);
  int count = 0;  // list length, meaningful in hg == 0 threads
  for (int c0 = 0; c0 < ncand_blk; c0 += kTC) {
    __syncthreads();
    for (int e = tid; e < G * kTC * D; e += kQB * G) {
      const int hh = e / (kTC * D), cc = (e / D) % kTC, ee = e % D;
      const int c = c0 + cc;
      kt[hh][cc][ee] = c < s.C ? k_sum[(((long long)b * s.Hq + g * G + hh) * s.C + c) * D + ee] : 0.f;
    }
    for (int e = tid; e < G * kTC; e += kQB * G) {
      const int c = c0 + e % kTC;
      bt[e / kTC][e % kTC] = c < s.C ? b_sum[((long long)b * s.Hq + g * G + e / kTC) * s.C + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 1
    for (int cc = 0; cc < kTC; ++cc) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < D; ++e) acc = fmaf(qr[e], kt[hg][cc][e], acc);
      st[qi][hg][cc] = acc * s.scale + bt[hg][cc];
    }
    __syncthreads();
    if (hg == 0) {
      for (int cc = 0; cc < kTC; ++cc) {
        const int c = c0 + cc;
        if (c >= ncand) break;
        float gv = st[qi][0][cc];
#pragma unroll
        for (int x = 1; x < G; ++x) gv = fmaxf(gv, st[qi][x][cc]);
        // sorted descending list; equal scores keep the earlier (smaller) chunk first
        if (count < s.K || gv > lg[qi][count - 1]) {
          int pos = count < s.K ? count : s.K - 1;
          while (pos > 0 && lg[qi][pos - 1] < gv) {
            lg[qi][pos] = lg[qi][pos - 1];
            lc[qi][pos] = lc[qi][pos - 1];
            --pos;
          }
          lg[qi][pos] = gv;
          lc[qi][pos] = c;
          if (count < s.K) ++count;
        }
      }
    }
  }
  __syncthreads();
  if (hg == 0 && valid) {
    // ascending chunk order
    for (int a = 1; a < count; ++a) {
      const int cv = lc[qi][a];
      int p = a;
      while (p > 0 && lc[qi][p - 1] > cv) {
        lc[qi][p] = lc[qi][p - 1];
        --p;
      }
      lc[qi][p] = cv;
    }
    for (int x = 0; x < s.K; ++x)
      idx[(((long long)b * s.Hkv + g) * s.N + i) * s.K + x] = x < count ? lc[qi][x] : -1;
  }
  __syncthreads();
  if (!valid) return;
  const int cnt = min(ncand, s.K);
  for (int x = 0; x < s.K; ++x) {
    float val = -INFINITY;
    if (x < cnt) {
      const int c = lc[qi][x];
      const float* kp = k_sum + (((long long)b * s.Hq + h) * s.C + c) * D;
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < D; ++e) acc = fmaf(qr[e], kp[e], acc);
      val = acc * s.scale + b_sum[((long long)b * s.Hq + h) * s.C + c];
    }
    s_sel[(((long long)b * s.Hq + h) * s.N + i) * s.K + x] = val;
  }
}

template <int D, int G>
cudaError_t go_prefill(const Shape& s, const void* q, const void* k_sum, const float* b_sum, int32_t* idx,
                       float* s_sel, cudaStream_t st) {
  dim3 grid((s.N + kQB - 1) / kQB, s.Hkv, s.B);
  if (s.K <= 64)
    score_topk_prefill_simt<D, G, 65><<<grid, kQB * G, 0, st>>>(s, (const float*)q, (const float*)k_sum, b_sum, idx,
                                                                 s_sel);
  else
    return cudaErrorNotSupported;
  return cudaGetLastError();
}

// ------------------------------------------------------------------ decode --
// Pass 1: per (b, group, chunk block) — s^ for every head and candidate,
// and the group max, written to the workspace.
template <typename T, int D, int G>
__global__ void __launch_bounds__(256) decode_scores(Shape s, const T* __restrict__ q, const T* __restrict__ k_sum,
                                                     const float* __restrict__ b_sum, float* __restrict__ s_all,
                                                     float* __restrict__ g_all, int ncand_max, DecView dv) {
  // lane layout: LPR lanes per (chunk, head) row (16 for d = 128: 8 elements each)
  constexpr int LPR = D / 8 >= 32 ? 32 : D / 8;  // lanes per row
  constexpr int EPL = D / LPR;                    // elements per lane
  constexpr int RPW = 32 / LPR;                   // rows per warp instruction
  // row groups per iteration: all their loads are issued before any is used,
  // so that each warp keeps U * G vectors per lane in flight
  constexpr int U = (sizeof(T) == 2 && EPL == 8) ? (G >= 8 ? 2 : 16 / G) : 1;
  __shared__ float qs[G][D];
  const int g = blockIdx.y, b = blockIdx.z;
  // candidates of this sequence's token at L - 1 (an out-of-range L has none)
  const int L = dv_len(dv, s, b);
  const int ncand = (L >= 1 && L <= s.N) ? min(ncand_max, max(0, (L - 1) / s.S - s.nw + 1)) : 0;
  for (int e = threadIdx.x; e < G * D; e += blockDim.x)
    qs[e / D][e % D] = to_f32(q[((long long)b * s.Hq + g * G + e / D) * D + e % D]);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int sub = lane / LPR, l = lane % LPR;
  const long long hrow = ((long long)b * s.Hq + g * G) * s.C;  // row of head g*G, chunk 0
  // the loop bound is warp-uniform so that every lane reaches the shuffles
  for (int cb = (blockIdx.x * nwarps + warp) * U * RPW; cb < ncand; cb += gridDim.x * nwarps * U * RPW) {
    if constexpr (sizeof(T) == 2 && EPL == 8) {
      uint4 u[U][G];
      float bs[U][G];
#pragma unroll
      for (int x = 0; x < U; ++x) {
        const int c = min(cb + x * RPW + sub, ncand - 1);  // rows past ncand re-read the last one
#pragma unroll
        for (int hg = 0; hg < G; ++hg) {
          u[x][hg] = __ldg(reinterpret_cast<const uint4*>(k_sum + (hrow + (long long)hg * s.C + c) * D + l * EPL));
          bs[x][hg] = __ldg(b_sum + hrow + (long long)hg * s.C + c);
        }
      }
#pragma unroll
      for (int x = 0; x < U; ++x) {
        const int c = cb + x * RPW + sub;
        const bool own = c < ncand;
        float gmax = -INFINITY;
#pragma unroll
        for (int hg = 0; hg < G; ++hg) {
          const uint32_t w[4] = {u[x][hg].x, u[x][hg].y, u[x][hg].z, u[x][hg].w};
          float acc = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = bf16x2_to_f32x2(w[e]);
            acc = fmaf(qs[hg][l * EPL + 2 * e], f.x, acc);
            acc = fmaf(qs[hg][l * EPL + 2 * e + 1], f.y, acc);
          }
#pragma unroll
          for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          const float sv = acc * s.scale + bs[x][hg];
          gmax = fmaxf(gmax, sv);
          if (l == 0 && own) s_all[hrow + (long long)hg * s.C + c] = sv;
        }
        if (l == 0 && own) g_all[((long long)b * s.Hkv + g) * s.C + c] = gmax;
      }
    } else {
      const int c = cb + sub < ncand ? cb + sub : cb;
      const bool own = cb + sub < ncand;
      float gmax = -INFINITY;
#pragma unroll
      for (int hg = 0; hg < G; ++hg) {
        const T* kp = k_sum + (hrow + (long long)hg * s.C + c) * D + l * EPL;
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc = fmaf(qs[hg][l * EPL + e], to_f32(kp[e]), acc);
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        const float sv = acc * s.scale + b_sum[hrow + (long long)hg * s.C + c];
        gmax = fmaxf(gmax, sv);
        if (l == 0 && own) s_all[hrow + (long long)hg * s.C + c] = sv;
      }
      if (l == 0 && own) g_all[((long long)b * s.Hkv + g) * s.C + c] = gmax;
    }
  }
}

// Pass 2: per (b, group) — exact top-K by radix select on the group scores.
// Keys are order-preserving uint32 images of the scores; ties at the
// threshold are broken toward smaller chunk indices with a prefix sum in
// chunk order, so the result does not depend on thread timing.
constexpr int kSelThreads = 1024;

template <int G>
__global__ void __launch_bounds__(kSelThreads) decode_select(Shape s, const float* __restrict__ s_all,
                                                             const float* __restrict__ g_all, int32_t* __restrict__ idx,
                                                             float* __restrict__ s_sel, int ncand_max, DecView dv,
                                                             DevCtx ctx) {
  __shared__ unsigned hist[256];
  __shared__ unsigned prefix_sh, need_sh;
  __shared__ int sel[64];
  __shared__ int nsel_sh;
  __shared__ unsigned scan[kSelThreads];
  const int g = blockIdx.x % s.Hkv, b = blockIdx.x / s.Hkv;
  const int tid = threadIdx.x;
  const int L = dv_len(dv, s, b);
  if ((L < 1 || L > s.N) && tid == 0) raise_status(ctx, kStatusBadIndex);
  const int ncand = (L >= 1 && L <= s.N) ? min(ncand_max, max(0, (L - 1) / s.S - s.nw + 1)) : 0;
  const float* gr = g_all + ((long long)b * s.Hkv + g) * s.C;
  const int K = s.K;
  if (tid == 0) nsel_sh = 0;
  __syncthreads();
  if (ncand <= K) {
    for (int c = tid; c < ncand; c += kSelThreads) sel[c] = c;
    if (tid == 0) nsel_sh = ncand;
  } else {
    // MSB-first radix select of the K-th largest key.  The bits above the
    // highest one in which the smallest and largest keys differ are common to
    // all keys, so the 8-bit digits start just below them: the scores of one
    // sequence span a narrow range and the leading digits would otherwise all
    // fall into one or two histogram bins.
    const int lane = tid & 31, wid = tid >> 5;
    unsigned kmin = 0xffffffffu, kmax = 0u;
    for (int c = tid; c < ncand; c += kSelThreads) {
      const unsigned key = float_key(gr[c]);
      kmin = min(kmin, key);
      kmax = max(kmax, key);
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
      scan[2 * wid] = kmin;
      scan[2 * wid + 1] = kmax;
    }
    __syncthreads();
    if (wid == 0) {
      unsigned a = lane < kSelThreads / 32 ? scan[2 * lane] : 0xffffffffu;
      unsigned z = lane < kSelThreads / 32 ? scan[2 * lane + 1] : 0u;
      a = __reduce_min_sync(0xffffffffu, a);
      z = __reduce_max_sync(0xffffffffu, z);
      if (lane == 0) {
        prefix_sh = a;
        need_sh = z;
      }
    }
    __syncthreads();
    const unsigned diff = prefix_sh ^ need_sh;
    const unsigned kmax_all = need_sh;
    __syncthreads();
    unsigned need = K;
    // bits above `top` are common to every key
    const int top = diff ? 31 - __clz(diff) : -1;
    unsigned prefix = top >= 31 ? 0u : (kmax_all & ~((2u << top) - 1u));
    for (int hi_bit = top; hi_bit >= 0; hi_bit -= 8) {
      const int shift = max(0, hi_bit - 7);
      const unsigned dmask = (2u << (hi_bit - shift)) - 1u;  // digit bits [shift, hi_bit]
      for (int x = tid; x < 256; x += kSelThreads) hist[x] = 0;
      __syncthreads();
      const unsigned hi_mask = hi_bit >= 31 ? 0u : (0xffffffffu << (hi_bit + 1));
      for (int c = tid; c < ncand; c += kSelThreads) {
        const unsigned key = float_key(gr[c]);
        if ((key & hi_mask) == (prefix & hi_mask)) atomicAdd(&hist[(key >> shift) & dmask], 1u);
      }
      __syncthreads();
      if (wid == 0) {
        // digit of the need-th largest key: lane l holds bins 8l .. 8l+7
        unsigned h8[8], own = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          h8[j] = hist[8 * lane + j];
          own += h8[j];
        }
        unsigned suf = own;  // keys in bins >= 8 lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned t = __shfl_down_sync(0xffffffffu, suf, o);
          if (lane + o < 32) suf += t;
        }
        const unsigned above = suf - own;  // keys in bins >= 8 (lane + 1)
        int digit = -1;
        unsigned acc = above;
        if (above < need && suf >= need) {
#pragma unroll
          for (int j = 7; j >= 0; --j) {
            if (digit < 0 && acc + h8[j] >= need) digit = j;
            else if (digit < 0) acc += h8[j];
          }
        }
        const unsigned who = __ballot_sync(0xffffffffu, digit >= 0);
        const int src = who ? __ffs(who) - 1 : 0;
        const int dg = __shfl_sync(0xffffffffu, 8 * lane + digit, src);
        const unsigned ac = __shfl_sync(0xffffffffu, acc, src);
        if (lane == 0) {
          prefix_sh = prefix | ((unsigned)dg << shift);
          need_sh = need - ac;
        }
      }
      __syncthreads();
      prefix = prefix_sh;
      need = need_sh;
      __syncthreads();
    }
    if (top < 0) prefix = kmax_all;  // all keys equal
    const unsigned thr = prefix;  // key of the K-th largest; `need` ties at thr are taken
    // strictly greater: order irrelevant (sorted afterwards)
    for (int c = tid; c < ncand; c += kSelThreads) {
      if (float_key(gr[c]) > thr) sel[atomicAdd(&nsel_sh, 1)] = c;
    }
    // ties: the `need` smallest chunk indices, via a prefix sum in chunk order
    const int per = (ncand + kSelThreads - 1) / kSelThreads;
    const int c_lo = tid * per, c_hi = min(ncand, c_lo + per);
    unsigned mine = 0;
    for (int c = c_lo; c < c_hi; ++c) mine += float_key(gr[c]) == thr;
    scan[tid] = mine;
    __syncthreads();
    for (int o = 1; o < kSelThreads; o <<= 1) {
      const unsigned v = tid >= o ? scan[tid - o] : 0u;
      __syncthreads();
      scan[tid] += v;
      __syncthreads();
    }
    unsigned rank = scan[tid] - mine;
    __syncthreads();
    const int base_gt = nsel_sh;
    for (int c = c_lo; c < c_hi; ++c) {
      if (float_key(gr[c]) == thr) {
        if (rank < need) sel[base_gt + rank] = c;
        ++rank;
      }
    }
    __syncthreads();
    if (tid == 0) nsel_sh = base_gt + (int)need;
  }
  __syncthreads();
  const int n = nsel_sh;
  // ascending order by rank counting (n <= 64)
  __shared__ int sorted[64];
  if (tid < n) {
    const int cv = sel[tid];
    int r = 0;
    for (int x = 0; x < n; ++x) r += sel[x] < cv;
    sorted[r] = cv;
  }
  __syncthreads();
  if (tid < K) {
    idx[((long long)b * s.Hkv + g) * K + tid] = tid < n ? sorted[tid] : -1;
  }
  for (int x = tid; x < G * K; x += kSelThreads) {
    const int hg = x / K, slot = x % K;
    const int h = g * G + hg;
    s_sel[((long long)b * s.Hq + h) * K + slot] =
        slot < n ? s_all[((long long)b * s.Hq + h) * s.C + sorted[slot]] : -INFINITY;
  }
}

template <typename T, int D, int G>
cudaError_t go_decode(const Shape& s, const void* q, const void* k_sum, const float* b_sum, int32_t* idx,
                      float* s_sel, void* ws, cudaStream_t st, const DevCtx& ctx, const DecView& dv) {
  const int cur = (s.N - 1) / s.S;
  const int ncand = max(0, cur - s.nw + 1);
  float* s_all = (float*)ws;
  float* g_all = s_all + (size_t)s.B * s.Hq * s.C;
  if (ncand > 0) {
    constexpr int LPR = D / 8 >= 32 ? 32 : D / 8;
    constexpr int U = (sizeof(T) == 2 && D / LPR == 8) ? (G >= 8 ? 2 : 16 / G) : 1;
    const int rows_per_block = 8 * U * (32 / LPR);
    int gx = (ncand + rows_per_block - 1) / rows_per_block;
    const int sms = device_sm_count();
    const int want = (sms * 8 + s.B * s.Hkv - 1) / (s.B * s.Hkv);
    if (gx > want) gx = want;
    decode_scores<T, D, G><<<dim3(gx, s.Hkv, s.B), 256, 0, st>>>(s, (const T*)q, (const T*)k_sum, b_sum, s_all,
                                                                  g_all, ncand, dv);
  }
  decode_select<G><<<s.B * s.Hkv, kSelThreads, 0, st>>>(s, s_all, g_all, idx, s_sel, ncand, dv, ctx);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t go_decode_g(const Shape& s, const void* q, const void* k_sum, const float* b_sum, int32_t* idx,
                        float* s_sel, void* ws, cudaStream_t st, const DevCtx& ctx, const DecView& dv) {
  switch (s.G) {
    case 1: return go_decode<T, D, 1>(s, q, k_sum, b_sum, idx, s_sel, ws, st, ctx, dv);
    case 2: return go_decode<T, D, 2>(s, q, k_sum, b_sum, idx, s_sel, ws, st, ctx, dv);
    case 4: return go_decode<T, D, 4>(s, q, k_sum, b_sum, idx, s_sel, ws, st, ctx, dv);
    case 8: return go_decode<T, D, 8>(s, q, k_sum, b_sum, idx, s_sel, ws, st, ctx, dv);
  }
  return cudaErrorNotSupported;
}

}  // namespace

cudaError_t launch_score_topk_simt(const Shape& s, const void* q, const void* k_sum, const float* b_sum, int32_t* idx,
                                   float* s_sel, cudaStream_t st, const DevCtx&) {
#define HILS_CASE(DD, GG) \
  if (s.d == DD && s.G == GG) return go_prefill<DD, GG>(s, q, k_sum, b_sum, idx, s_sel, st);
  HILS_CASE(32, 1) HILS_CASE(32, 2) HILS_CASE(32, 4) HILS_CASE(32, 8)
  HILS_CASE(64, 1) HILS_CASE(64, 2) HILS_CASE(64, 4) HILS_CASE(64, 8)
  HILS_CASE(128, 1) HILS_CASE(128, 2) HILS_CASE(128, 4)
#undef HILS_CASE
  return cudaErrorNotSupported;
}

size_t decode_score_workspace(const Shape& s) {
  return ((size_t)s.B * s.Hq * s.C + (size_t)s.B * s.Hkv * s.C) * sizeof(float);
}

cudaError_t launch_score_topk_decode(const Shape& s, const void* q, const void* k_sum, const float* b_sum,
                                     int32_t* idx, float* s_sel, void* ws, cudaStream_t st, const DevCtx& ctx,
                                     const DecView& dv) {
  if (s.dtype == 0) {
    if (s.d == 32) return go_decode_g<float, 32>(s, q, k_sum, b_sum, idx, s_sel, ws, st, ctx, dv);
    if (s.d == 64) return go_decode_g<float, 64>(s, q, k_sum, b_sum, idx, s_sel, ws, st, ctx, dv);
    if (s.d == 128) return go_decode_g<float, 128>(s, q, k_sum, b_sum, idx, s_sel, ws, st, ctx, dv);
  } else {
    if (s.d == 128) return go_decode_g<__nv_bfloat16, 128>(s, q, k_sum, b_sum, idx, s_sel, ws, st, ctx, dv);
  }
  return cudaErrorNotSupported;
}

}  // namespace hils
