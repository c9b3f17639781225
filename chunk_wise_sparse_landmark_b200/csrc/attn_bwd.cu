// Backward pass of the HiLS prefill: gradients of the attention output with
// respect to q, k, v and the landmark queries q'_c, with the chunk selection
// held fixed (top-K is a discrete choice).
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method): the token weight factorises as
//   w_ij = exp(s_ij)/Z_{i,c(j)} * exp(s^_{i,c(j)}) / Z^_i,
//   Z^_i = sum_{c in I_i} exp(s^_{i,c}) + Z_{i,swa},
// so the loss reaches the chunk scores s^ = q.k'/sqrt(d) + b' through the
// fusion weights, and from them the landmark summaries k', b' and their
// queries q'_c (the wmrh.cn article: the hierarchical softmax lets the
// language-model loss train the summaries).  With w_u = e^{A_u}/Z^ for the
// window unit and every chosen chunk (A_c = s^_c), out = sum_u w_u O_u and
// D = dout.out = sum_u w_u X_u with X_u = dout.O_u:
//   window key j:        omega_j = e^{s_ij}/Z^,     ds_ij = omega_j (dout.v_j - D)
//   chosen chunk c, j:   ds_ij = w_c p_j (dout.v_j - X_c)      (p: the chunk's own softmax)
//                        dA_c  = w_c (X_c - D)
//   dv_j += (weight of j) dout,  dq_i += scale sum_j ds_ij k_j,  dk_j += scale ds_ij q_i
//   score:     dq_i += scale sum_c dA_c k'_c,  dk'_c += scale dA_c q_i,  db'_c += dA_c
//   summaries: dp_j = dk'.k_j - db' (log p_j + 1),  dl_j = p_j (dp_j - sum_m p_m dp_m),
//              dk_j += p_j dk' + scale dl_j q'_c,   dq'_c = scale sum_j dl_j k_j
//
// Two kernels on CUDA cores (fp32 arithmetic, every input widened exactly):
//   bwd_rows_kernel  one warp per (sequence, query head, position): recomputes
//                    the row's logits, dout.v_j, the window and chunk masses
//                    and Z^, then writes dq (attention and score paths), dA
//                    per chosen slot, and the row statistics the second kernel
//                    needs (log Z^, D; per slot w_c, X_c).
//   bwd_keys_kernel  one CTA per (sequence, KV group, chunk): every key row of
//                    the chunk belongs to it alone, so its dk and dv are summed
//                    in registers over the rows that chose the chunk (bucket
//                    lists, grouped by chunk like the forward's chunk-major
//                    pass) and the window rows that see it; then the chunk's
//                    score and summary gradients (dk', db' -> dk, dq') for the
//                    G heads.  No floating-point atomics on global memory; the
//                    rows of a chunk are summed in the order of its bucket list,
//                    which the scatter fills by atomic arrival, so dk, dv and
//                    dq' repeat to fp32 rounding (dq and dA bit for bit).
// A thread of bwd_keys_kernel owns one key row j and a quarter of the head
// dimension, and keeps that key's k, v and accumulators in registers.
#include <algorithm>

#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int kRowWarps = 4;   // rows per block of bwd_rows_kernel
constexpr int kBatch = 4;      // rows per step of bwd_keys_kernel

template <typename T>
HILS_DI float ld(const T* p) {
  return to_f32(*p);
}

// ----------------------------------------------------------- bucketing ----
// Selection pairs grouped by (sequence, KV group, chunk), over all positions:
// entry (position << 6 | slot); the same acceptance rule as the forward.
__global__ void bwd_count_kernel(Shape s, const int32_t* __restrict__ idx, int* __restrict__ cnt, DevCtx ctx) {
  const long long lists = (long long)s.B * s.Hkv * s.N;
  const long long wpb = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (long long r = blockIdx.x * wpb + (threadIdx.x >> 5); r < lists; r += (long long)gridDim.x * wpb) {
    const int p = (int)(r % s.N);
    const long long bg = r / s.N;
    const int32_t* L = idx + r * s.K;
    int a = lane < s.K ? __ldg(L + lane) : -1, b = lane + 32 < s.K ? __ldg(L + lane + 32) : -1;
    bool bad;
    accept_list_warp(a, b, s.K, max(0, p / s.S - s.nw + 1), bad);
    if (bad && lane == 0) raise_status(ctx, kStatusBadIndex);
    if (a >= 0) atomicAdd(cnt + bg * s.C + a, 1);
    if (b >= 0) atomicAdd(cnt + bg * s.C + b, 1);
  }
}

// one block: exclusive scan of the bucket counts; cnt becomes the scatter cursor
__global__ void __launch_bounds__(1024) bwd_scan_kernel(int U, int* __restrict__ cnt, int* __restrict__ off) {
  __shared__ int wsum[32];
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int per = (U + 1023) / 1024;
  const int u0 = min(U, t * per), u1 = min(U, u0 + per);
  int sum = 0;
  for (int u = u0; u < u1; ++u) sum += cnt[u];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) wsum[w] = incl;
  __syncthreads();
  if (w == 0) {
    int x = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    wsum[lane] = x;
  }
  __syncthreads();
  int run = incl - sum + (w > 0 ? wsum[w - 1] : 0);
  for (int u = u0; u < u1; ++u) {
    const int n = cnt[u];
    off[u] = run;
    cnt[u] = run;
    run += n;
  }
  if (t == 1023) off[U] = run;
}

__global__ void bwd_scatter_kernel(Shape s, const int32_t* __restrict__ idx, int* __restrict__ cur,
                                   int* __restrict__ ent) {
  const long long lists = (long long)s.B * s.Hkv * s.N;
  const long long wpb = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (long long r = blockIdx.x * wpb + (threadIdx.x >> 5); r < lists; r += (long long)gridDim.x * wpb) {
    const int p = (int)(r % s.N);
    const long long bg = r / s.N;
    const int32_t* L = idx + r * s.K;
    int a = lane < s.K ? __ldg(L + lane) : -1, b = lane + 32 < s.K ? __ldg(L + lane + 32) : -1;
    bool bad;
    accept_list_warp(a, b, s.K, max(0, p / s.S - s.nw + 1), bad);
    if (a >= 0) ent[atomicAdd(cur + bg * s.C + a, 1)] = (p << 6) | lane;
    if (b >= 0) ent[atomicAdd(cur + bg * s.C + b, 1)] = (p << 6) | (lane + 32);
  }
}

// ------------------------------------------------------------- rows -------
// Per-warp scratch: logits and dout.v of the row's window keys and chosen
// chunks (cap = W + K S each), then per slot A_c, X_c, LSE_c.
template <typename T, int D>
__global__ void __launch_bounds__(32 * kRowWarps) bwd_rows_kernel(
    Shape s, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ k_sum,
    const int32_t* __restrict__ idx, const float* __restrict__ s_sel, const T* __restrict__ dout,
    float* __restrict__ dq, float* __restrict__ ds_sel, float2* __restrict__ st_row, float2* __restrict__ st_slot,
    int cap) {
  constexpr int E = D / 32;
  extern __shared__ float smem[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * kRowWarps + wib;
  const long long rows = (long long)s.B * s.Hq * s.N;
  if (row >= rows) return;
  const int i = (int)(row % s.N), h = (int)((row / s.N) % s.Hq), b = (int)(row / ((long long)s.N * s.Hq));
  const int g = h / s.G, K = s.K;
  float* ls = smem + (size_t)wib * (2 * cap + 3 * 64);
  float* lg = ls + cap;
  float* sA = lg + cap;
  float* sX = sA + 64;
  float* sL = sX + 64;
  float qr[E], gr[E];
#pragma unroll
  for (int t = 0; t < E; ++t) {
    qr[t] = ld(q + row * D + lane + 32 * t);
    gr[t] = ld(dout + row * D + lane + 32 * t);
  }
  const T* kb = k + ((long long)b * s.Hkv + g) * s.N * D;
  const T* vb = v + ((long long)b * s.Hkv + g) * s.N * D;
  auto dots = [&](int key, float& sv, float& gv) {
    float a = 0.f, c = 0.f;
#pragma unroll
    for (int t = 0; t < E; ++t) {
      a = fmaf(qr[t], ld(kb + (long long)key * D + lane + 32 * t), a);
      c = fmaf(gr[t], ld(vb + (long long)key * D + lane + 32 * t), c);
    }
    sv = warp_sum(a) * s.scale;
    gv = warp_sum(c);
  };
  // window keys [w0, i]
  const int cur = i / s.S;
  const int w0 = max(0, (cur - s.nw + 1) * s.S), nwin = i - w0 + 1;
  float mw = -INFINITY;
  for (int j = 0; j < nwin; ++j) {
    float sv, gv;
    dots(w0 + j, sv, gv);
    if (lane == 0) {
      ls[j] = sv;
      lg[j] = gv;
    }
    mw = fmaxf(mw, sv);
  }
  __syncwarp();
  float lw = 0.f, xw = 0.f;
  for (int j = lane; j < nwin; j += 32) {
    const float e = expf(ls[j] - mw);
    lw += e;
    xw += e * lg[j];
  }
  lw = warp_sum(lw);
  xw = warp_sum(xw);
  const float a_swa = mw + logf(lw), x_swa = xw / lw;
  // chosen chunks (the list form, common.cuh)
  const int ncand = max(0, cur - s.nw + 1);
  const int32_t* ir = idx + (((long long)b * s.Hkv + g) * s.N + i) * K;
  const float* sr = s_sel + row * K;
  float M = a_swa;
  uint64_t okm = 0ull;
  int prev = -1;
  for (int x = 0; x < K; ++x) {
    const int c = __ldg(ir + x);
    const bool ok = c >= 0 && c < ncand && c > prev;
    prev = c < 0 ? 0x7fffffff : max(prev, c);
    if (!ok) continue;
    okm |= 1ull << x;
    float* lsx = ls + nwin + x * s.S;
    float* lgx = lg + nwin + x * s.S;
    float mc = -INFINITY;
    for (int j = 0; j < s.S; ++j) {
      float sv, gv;
      dots(c * s.S + j, sv, gv);
      if (lane == 0) {
        lsx[j] = sv;
        lgx[j] = gv;
      }
      mc = fmaxf(mc, sv);
    }
    __syncwarp();
    float lc = 0.f, xc = 0.f;
    for (int j = lane; j < s.S; j += 32) {
      const float e = expf(lsx[j] - mc);
      lc += e;
      xc += e * lgx[j];
    }
    lc = warp_sum(lc);
    xc = warp_sum(xc);
    const float A = __ldg(sr + x);
    M = fmaxf(M, A);
    if (lane == 0) {
      sA[x] = A;
      sX[x] = xc / lc;
      sL[x] = mc + logf(lc);
    }
  }
  __syncwarp();
  float zhat = expf(a_swa - M);
  for (int x = 0; x < K; ++x)
    if (okm >> x & 1ull) zhat += expf(sA[x] - M);
  const float lz = M + logf(zhat);
  float Dv = expf(a_swa - lz) * x_swa;
  for (int x = 0; x < K; ++x)
    if (okm >> x & 1ull) Dv += expf(sA[x] - lz) * sX[x];
  // dq: window keys, then chosen chunks (attention logits and score path)
  float dqr[E];
#pragma unroll
  for (int t = 0; t < E; ++t) dqr[t] = 0.f;
  for (int j = 0; j < nwin; ++j) {
    const float ds = expf(ls[j] - lz) * (lg[j] - Dv);
#pragma unroll
    for (int t = 0; t < E; ++t) dqr[t] = fmaf(ds, ld(kb + (long long)(w0 + j) * D + lane + 32 * t), dqr[t]);
  }
  const T* ksr = k_sum + ((long long)b * s.Hq + h) * s.C * D;
  for (int x = 0; x < K; ++x) {
    float dA = 0.f, wc = 0.f;
    if (okm >> x & 1ull) {
      const int c = __ldg(ir + x);
      wc = expf(sA[x] - lz);
      dA = wc * (sX[x] - Dv);
      const float* lsx = ls + nwin + x * s.S;
      const float* lgx = lg + nwin + x * s.S;
      for (int j = 0; j < s.S; ++j) {
        const float ds = wc * expf(lsx[j] - sL[x]) * (lgx[j] - sX[x]);
#pragma unroll
        for (int t = 0; t < E; ++t) dqr[t] = fmaf(ds, ld(kb + (long long)(c * s.S + j) * D + lane + 32 * t), dqr[t]);
      }
#pragma unroll
      for (int t = 0; t < E; ++t) dqr[t] = fmaf(dA, ld(ksr + (long long)c * D + lane + 32 * t), dqr[t]);
    }
    if (lane == 0) {
      ds_sel[row * K + x] = dA;
      st_slot[row * K + x] = make_float2(wc, (okm >> x & 1ull) ? sX[x] : 0.f);
    }
  }
#pragma unroll
  for (int t = 0; t < E; ++t) dq[row * D + lane + 32 * t] = dqr[t] * s.scale;
  if (lane == 0) st_row[row] = make_float2(lz, Dv);
}

// ------------------------------------------------------------- keys -------
// One CTA per (sequence, KV group, chunk c) with 4 S threads: thread t owns
// key row j = t / 4 and the quarter qt = t % 4 of the head dimension.  Rows
// are taken kBatch at a time: the chosen rows (bucket pairs x G heads), then
// the window rows (positions whose window holds chunk c, x G heads).
template <typename T, int D>
__global__ void __launch_bounds__(256) bwd_keys_kernel(
    Shape s, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const T* __restrict__ q_lmk, const T* __restrict__ dout, const int* __restrict__ off,
    const int* __restrict__ ent, const float* __restrict__ ds_sel, const float2* __restrict__ st_row,
    const float2* __restrict__ st_slot, float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dq_lmk) {
  constexpr int Q4 = D / 4;
  __shared__ float sq[kBatch][D], sg[kBatch][D];
  __shared__ float sred[8][kBatch], sred2[8][kBatch];
  __shared__ float sdks[8][D], sdbs[8];
  __shared__ float sqp[D], sdq[D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int j = tid >> 2, qt = tid & 3;
  const int nchunks_all = (s.N + s.S - 1) / s.S;
  const int c = blockIdx.x % nchunks_all;
  const long long bg = blockIdx.x / nchunks_all;
  const int b = (int)(bg / s.Hkv), g = (int)(bg % s.Hkv);
  const int key = c * s.S + j;
  const bool kvalid = key < s.N;
  const long long kvoff = (bg * s.N + (kvalid ? key : 0)) * D + qt * Q4;
  float kr[Q4], vr[Q4], dka[Q4], dva[Q4];
#pragma unroll
  for (int e = 0; e < Q4; ++e) {
    kr[e] = kvalid ? ld(k + kvoff + e) : 0.f;
    vr[e] = kvalid ? ld(v + kvoff + e) : 0.f;
    dka[e] = dva[e] = 0.f;
  }
  for (int x = tid; x < 8 * D; x += blockDim.x) sdks[x / D][x % D] = 0.f;
  if (tid < 8) sdbs[tid] = 0.f;
  const bool complete = c < s.C;
  const int u = (int)(bg * s.C + c);
  const int n_sel = complete ? (__ldg(off + u + 1) - __ldg(off + u)) * s.G : 0;
  const int p_lo = c * s.S, p_hi = min(s.N, (c + s.nw) * s.S);
  const int n_win = (p_hi - p_lo) * s.G;
  const int n_rows = n_sel + n_win;
  __syncthreads();
  for (int r0 = 0; r0 < n_rows; r0 += kBatch) {
    // rows of this step: (position, head, chosen slot or -1)
    int rp[kBatch], rh[kBatch], rx[kBatch];
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      const int rr = r0 + r;
      rp[r] = -1;
      rh[r] = 0;
      rx[r] = -1;
      if (rr < n_sel) {
        const int e = __ldg(ent + __ldg(off + u) + rr / s.G);
        rp[r] = e >> 6;
        rx[r] = e & 63;
        rh[r] = g * s.G + rr % s.G;
      } else if (rr < n_rows) {
        const int w = rr - n_sel;
        rp[r] = p_lo + w / s.G;
        rh[r] = g * s.G + w % s.G;
      }
    }
    for (int x = tid; x < kBatch * D; x += blockDim.x) {
      const int r = x / D, e = x % D;
      const long long qrow = (((long long)b * s.Hq + rh[r]) * s.N + max(rp[r], 0)) * D;
      sq[r][e] = rp[r] >= 0 ? ld(q + qrow + e) : 0.f;
      sg[r][e] = rp[r] >= 0 ? ld(dout + qrow + e) : 0.f;
    }
    __syncthreads();
    float sv[kBatch], gv[kBatch];
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      float a = 0.f, cc = 0.f;
#pragma unroll
      for (int e = 0; e < Q4; ++e) {
        a = fmaf(sq[r][qt * Q4 + e], kr[e], a);
        cc = fmaf(sg[r][qt * Q4 + e], vr[e], cc);
      }
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      cc += __shfl_xor_sync(0xffffffffu, cc, 1);
      cc += __shfl_xor_sync(0xffffffffu, cc, 2);
      sv[r] = a * s.scale;
      gv[r] = cc;
      // causal: a window row of the chunk's own positions sees keys <= itself
      const bool seen = kvalid && rp[r] >= 0 && (rx[r] >= 0 || key <= rp[r]);
      if (!seen) sv[r] = -INFINITY;
    }
    // the chunk's own log-mass for chosen rows: max and sum over the S keys
    float mx[kBatch];
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      float m = warp_max(sv[r]);
      if (lane == 0) sred[warp][r] = m;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      float m = -INFINITY;
      for (int w = 0; w < nwarps; ++w) m = fmaxf(m, sred[w][r]);
      mx[r] = m;
      // each key is held by 4 threads: count it once
      float z = (qt == 0 && sv[r] != -INFINITY) ? expf(sv[r] - m) : 0.f;
      z = warp_sum(z);
      if (lane == 0) sred2[warp][r] = z;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      if (rp[r] < 0) continue;
      const long long hrow = ((long long)b * s.Hq + rh[r]) * s.N + rp[r];
      float wgt, ds;
      if (rx[r] >= 0) {
        float z = 0.f;
        for (int w = 0; w < nwarps; ++w) z += sred2[w][r];
        const float2 wx = __ldg(st_slot + hrow * s.K + rx[r]);
        const float p = sv[r] == -INFINITY ? 0.f : expf(sv[r] - mx[r]) / z;
        wgt = wx.x * p;
        ds = wgt * (gv[r] - wx.y);
      } else {
        const float2 zd = __ldg(st_row + hrow);
        wgt = sv[r] == -INFINITY ? 0.f : expf(sv[r] - zd.x);
        ds = wgt * (gv[r] - zd.y);
      }
#pragma unroll
      for (int e = 0; e < Q4; ++e) {
        dka[e] = fmaf(ds * s.scale, sq[r][qt * Q4 + e], dka[e]);
        dva[e] = fmaf(wgt, sg[r][qt * Q4 + e], dva[e]);
      }
    }
    // score path of the chosen rows: dk'_h += scale dA q, db'_h += dA
    for (int e = tid; e < D; e += blockDim.x) {
#pragma unroll
      for (int r = 0; r < kBatch; ++r) {
        if (rp[r] < 0 || rx[r] < 0) continue;
        const long long hrow = ((long long)b * s.Hq + rh[r]) * s.N + rp[r];
        const float dA = __ldg(ds_sel + hrow * s.K + rx[r]);
        const int hg = rh[r] - g * s.G;
        sdks[hg][e] = fmaf(dA * s.scale, sq[r][e], sdks[hg][e]);
        if (e == 0) sdbs[hg] += dA;
      }
    }
    __syncthreads();
  }
  // summaries of the G heads of this chunk (complete chunks only)
  if (complete) {
    for (int hg = 0; hg < s.G; ++hg) {
      const int h = g * s.G + hg;
      const long long t = ((long long)b * s.Hq + h) * s.C + c;
      for (int e = tid; e < D; e += blockDim.x) {
        sqp[e] = ld(q_lmk + t * D + e);
        sdq[e] = 0.f;
      }
      __syncthreads();
      float a = 0.f, uu = 0.f;
#pragma unroll
      for (int e = 0; e < Q4; ++e) {
        a = fmaf(sqp[qt * Q4 + e], kr[e], a);
        uu = fmaf(sdks[hg][qt * Q4 + e], kr[e], uu);
      }
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      uu += __shfl_xor_sync(0xffffffffu, uu, 1);
      uu += __shfl_xor_sync(0xffffffffu, uu, 2);
      const float l = a * s.scale;
      float m = warp_max(l);
      if (lane == 0) sred[warp][0] = m;
      __syncthreads();
      m = -INFINITY;
      for (int w = 0; w < nwarps; ++w) m = fmaxf(m, sred[w][0]);
      float z = qt == 0 ? expf(l - m) : 0.f;
      z = warp_sum(z);
      if (lane == 0) sred2[warp][0] = z;
      __syncthreads();
      z = 0.f;
      for (int w = 0; w < nwarps; ++w) z += sred2[w][0];
      const float lp = l - m - logf(z), p = expf(lp);
      const float dp = uu - sdbs[hg] * (lp + 1.f);
      float pdp = qt == 0 ? p * dp : 0.f;
      pdp = warp_sum(pdp);
      __syncthreads();  // sred[.][1] reuse is safe: everyone has read sred2
      if (lane == 0) sred[warp][1] = pdp;
      __syncthreads();
      pdp = 0.f;
      for (int w = 0; w < nwarps; ++w) pdp += sred[w][1];
      const float dl = p * (dp - pdp);
#pragma unroll
      for (int e = 0; e < Q4; ++e) {
        dka[e] = fmaf(p, sdks[hg][qt * Q4 + e], dka[e]);
        dka[e] = fmaf(dl * s.scale, sqp[qt * Q4 + e], dka[e]);
        atomicAdd(&sdq[qt * Q4 + e], dl * s.scale * kr[e]);  // shared memory
      }
      __syncthreads();
      for (int e = tid; e < D; e += blockDim.x) dq_lmk[t * D + e] = sdq[e];
      __syncthreads();
    }
  }
  if (kvalid) {
#pragma unroll
    for (int e = 0; e < Q4; ++e) {
      dk[kvoff + e] = dka[e];
      dv[kvoff + e] = dva[e];
    }
  }
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdWs {
  size_t cnt, off, ent, st_row, st_slot, ds, total;
};

BwdWs bwd_ws(const Shape& s) {
  BwdWs w{};
  const size_t U = (size_t)s.B * s.Hkv * s.C;
  const size_t rows = (size_t)s.B * s.Hq * s.N;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o += up256(bytes);
    return r;
  };
  w.cnt = take((U + 1) * 4);
  w.off = take((U + 1) * 4);
  w.ent = take((size_t)s.B * s.Hkv * s.N * s.K * 4);
  w.st_row = take(rows * 8);
  w.st_slot = take(rows * s.K * 8);
  w.ds = take(rows * s.K * 4);
  w.total = o;
  return w;
}

template <typename T, int D>
cudaError_t go_bwd(const Shape& s, const void* q, const void* k, const void* v, const void* q_lmk, const int32_t* idx,
                   const float* s_sel, const void* k_sum, const void* dout, float* dq, float* dk, float* dv,
                   float* dq_lmk, float* ds_sel, void* ws, cudaStream_t st, const DevCtx& ctx) {
  const BwdWs w = bwd_ws(s);
  unsigned char* W = (unsigned char*)ws;
  int* cnt = (int*)(W + w.cnt);
  int* off = (int*)(W + w.off);
  int* ent = (int*)(W + w.ent);
  float2* st_row = (float2*)(W + w.st_row);
  float2* st_slot = (float2*)(W + w.st_slot);
  float* ds = ds_sel ? ds_sel : (float*)(W + w.ds);
  const int U = s.B * s.Hkv * s.C;
  const int sms = device_sm_count();
  cudaError_t e = cudaMemsetAsync(cnt, 0, (size_t)(U + 1) * 4, st);
  if (e != cudaSuccess) return e;
  const long long lists = (long long)s.B * s.Hkv * s.N;
  const int grid = (int)std::min<long long>((lists + 7) / 8, (long long)sms * 16);
  if (U > 0) {
    bwd_count_kernel<<<grid, 256, 0, st>>>(s, idx, cnt, ctx);
    bwd_scan_kernel<<<1, 1024, 0, st>>>(U, cnt, off);
    bwd_scatter_kernel<<<grid, 256, 0, st>>>(s, idx, cnt, ent);
  } else {
    e = cudaMemsetAsync(off, 0, 4, st);
    if (e != cudaSuccess) return e;
  }
  const int cap = s.W + s.K * s.S;
  const size_t smem = (size_t)kRowWarps * (2 * cap + 3 * 64) * sizeof(float);
  e = ensure_dynamic_smem((const void*)bwd_rows_kernel<T, D>, (int)smem);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)s.B * s.Hq * s.N;
  bwd_rows_kernel<T, D><<<(unsigned)((rows + kRowWarps - 1) / kRowWarps), 32 * kRowWarps, smem, st>>>(
      s, (const T*)q, (const T*)k, (const T*)v, (const T*)k_sum, idx, s_sel, (const T*)dout, dq, ds, st_row, st_slot,
      cap);
  const long long ctas = (long long)s.B * s.Hkv * ((s.N + s.S - 1) / s.S);
  bwd_keys_kernel<T, D><<<(unsigned)ctas, 4 * s.S, 0, st>>>(s, (const T*)q, (const T*)k, (const T*)v,
                                                             (const T*)q_lmk, (const T*)dout, off, ent, ds, st_row,
                                                             st_slot, dk, dv, dq_lmk);
  return cudaGetLastError();
}

}  // namespace

size_t prefill_bwd_workspace(const Shape& s) { return bwd_ws(s).total; }

cudaError_t launch_prefill_bwd(const Shape& s, const void* q, const void* k, const void* v, const void* q_lmk,
                               const int32_t* idx, const float* s_sel, const void* k_sum, const void* dout, float* dq,
                               float* dk, float* dv, float* dq_lmk, float* ds_sel, void* ws, cudaStream_t st,
                               const DevCtx& ctx) {
  if (s.S > 64 || s.K > 64 || s.G > 8) return cudaErrorNotSupported;
  if (s.dtype == 0) {
    if (s.d == 32) return go_bwd<float, 32>(s, q, k, v, q_lmk, idx, s_sel, k_sum, dout, dq, dk, dv, dq_lmk, ds_sel, ws, st, ctx);
    if (s.d == 64) return go_bwd<float, 64>(s, q, k, v, q_lmk, idx, s_sel, k_sum, dout, dq, dk, dv, dq_lmk, ds_sel, ws, st, ctx);
    if (s.d == 128) return go_bwd<float, 128>(s, q, k, v, q_lmk, idx, s_sel, k_sum, dout, dq, dk, dv, dq_lmk, ds_sel, ws, st, ctx);
  } else if (s.d == 128) {
    return go_bwd<__nv_bfloat16, 128>(s, q, k, v, q_lmk, idx, s_sel, k_sum, dout, dq, dk, dv, dq_lmk, ds_sel, ws, st,
                                      ctx);
  }
  return cudaErrorNotSupported;
}

}  // namespace hils
