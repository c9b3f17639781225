// Hierarchical-softmax sparse attention for decode (one new token per
// sequence), split across CTAs.
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method): token weight w_{i,j} = exp(s_ij)/Z_{i,c(j)} * exp(s^_{i,c(j)})/Z^_i,
// Z^_i = sum_c exp(s^_{i,c}) + Z_{i,swa}; section 实验 (Experiments) reports
// sublinear decode latency — the token touches only its K chunks and its
// window.
//
// Work unit = one 64-key (S-key) tile: either a selected chunk or one chunk of
// the window.  Per (sequence, KV group) the K + n_w units are dealt to
// `nsplit` CTAs; each CTA serves all G query heads of the group, so every key
// and value tile is read from HBM exactly once.  A unit contributes
// e^{a} * o to the numerator and e^{a} * z to the denominator, where for a
// selected chunk a = s^ - log l, z = l, and for a window tile a = m, z = l
// (m = tile max, l = sum e^{s-m}, o = sum e^{s-m} v).  Each CTA folds its units
// with a running maximum and writes one (M, den, num[d]) record per head to the
// workspace; a second kernel folds the records of a head and divides.
// Tiles arrive through 1-D bulk copies (TMA) into a two-stage shared-memory
// ring; every wait is bounded.
#include <mutex>

#include "gather_mma.cuh"
#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int kThreads = 256;

template <typename T, int D, int S, int G>
struct DecSmem {
  alignas(128) T kt[2][S * D];
  alignas(128) T vt[2][S * D];
  float qs[G][D];
  float p[G][S];
  float a[G], z[G];
  uint64_t full[2];
};

// shared-memory position of element e of key row j, rotated so that the 16-byte
// vectors of consecutive rows start in different banks
template <typename T, int D>
HILS_DI const T* row_ptr(const T* tile, int j) { return tile + j * D; }

template <typename T, int D, int S, int G>
__global__ void __launch_bounds__(kThreads) attn_decode_partial(Shape s, const T* __restrict__ q,
                                                                const T* __restrict__ k, const T* __restrict__ v,
                                                                const int32_t* __restrict__ idx,
                                                                const float* __restrict__ s_sel,
                                                                float* __restrict__ ws, int nsplit, DecView dv, DevCtx ctx) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  auto& sm = *reinterpret_cast<DecSmem<T, D, S, G>*>(smem_raw);
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int L = dv_len(dv, s, b);
  const bool len_ok = L >= 1 && L <= s.N;  // invalid: reported, no units (the record stays empty)
  if (!len_ok) {
    if (tid == 0) raise_status(ctx, kStatusBadIndex);
    L = 1;
  }
  const int pos = L - 1, cur = pos / S;
  const int ncand = max(0, cur - s.nw + 1);
  const int wc0 = max(0, cur - s.nw + 1);        // first window chunk
  const int nwin = cur - wc0 + 1;                 // window tiles
  const int nunits = len_ok ? s.K + nwin : 0;
  const int32_t* ir = idx + ((long long)b * s.Hkv + g) * s.K;

  for (int e = tid; e < G * D; e += kThreads)
    sm.qs[e / D][e % D] = to_f32(q[((long long)b * s.Hq + g * G + e / D) * D + e % D]);
  if (tid == 0) {
    mbar_init(&sm.full[0], 1);
    mbar_init(&sm.full[1], 1);
    fence_barrier_init();
  }
  __syncthreads();

  // this CTA's units: u = split, split + nsplit, ... ; resolve each to a key range
  auto unit_keys = [&](int u, long long& off, int& nk, bool& sel, int& slot) -> bool {
    if (u < s.K) {
      const int c = ir[u];
      sel = true;
      slot = u;
      if (!list_entry_accepted(ir, u, ncand)) {  // the list form, common.cuh
        if (c != -1 && tid == 0) raise_status(ctx, kStatusBadIndex);
        return false;
      }
      off = dv_chunk(dv, s, b, g, c);
      nk = S;
    } else {
      const int wc = wc0 + (u - s.K);
      sel = false;
      slot = -1;
      off = dv_chunk(dv, s, b, g, wc);
      nk = min(S, L - wc * S);
    }
    if (off < 0) {  // a page outside the pool: reported, never read
      if (tid == 0) raise_status(ctx, kStatusBadIndex);
      return false;
    }
    return true;
  };
  bool inflight[2] = {false, false};  // meaningful in thread 0
  auto issue = [&](int stage, long long off, int nk) {
    if (ctx.inject == 1) return;  // test hook: no copy, the wait below must run out
    inflight[stage] = true;
    fence_proxy_async_shared();
    const uint32_t bytes = (uint32_t)(nk * D * sizeof(T));
    mbar_arrive_expect_tx(&sm.full[stage], 2 * bytes);
    tma_load_1d(sm.kt[stage], k + off, bytes, &sm.full[stage]);
    tma_load_1d(sm.vt[stage], v + off, bytes, &sm.full[stage]);
  };

  // running fold per head, thread (h, e) owns num for dims e, e + 128 ... via loop
  float Mh[G], den[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    Mh[h] = -INFINITY;
    den[h] = 0.f;
  }
  constexpr int OUTS = (G * D + kThreads - 1) / kThreads;  // outputs per thread
  float num[OUTS];
#pragma unroll
  for (int r = 0; r < OUTS; ++r) num[r] = 0.f;

  // collect the list of live units first (uniform across the CTA)
  int ulist[16];
  int nu = 0;
  for (int u = split; u < nunits && nu < 16; u += nsplit) {
    long long j0;
    int nk, slot;
    bool sel;
    if (unit_keys(u, j0, nk, sel, slot)) ulist[nu++] = u;
  }
  uint32_t phase[2] = {0u, 0u};
  if (tid == 0 && nu > 0) {
    long long j0;
    int nk, slot;
    bool sel;
    unit_keys(ulist[0], j0, nk, sel, slot);
    issue(0, j0, nk);
  }
  bool alive = true;  // CTA-wide: every thread sees the same value
  for (int x = 0; x < nu; ++x) {
    const int stage = x & 1;
    long long j0;
    int nk, slot;
    bool sel;
    unit_keys(ulist[x], j0, nk, sel, slot);
    if (tid == 0 && x + 1 < nu) {
      long long j0n;
      int nkn, sln;
      bool seln;
      unit_keys(ulist[x + 1], j0n, nkn, seln, sln);
      issue(stage ^ 1, j0n, nkn);
    }
    const bool landed = mbar_wait(&sm.full[stage], phase[stage], ctx);
    if (landed) inflight[stage] = false;
    phase[stage] ^= 1u;
    if (!__syncthreads_and(landed)) {
      alive = false;
      break;
    }
    // logits: thread per (h, j)
    for (int p = tid; p < G * S; p += kThreads) {
      const int h = p / S, j = p % S;
      float acc = -INFINITY;
      if (j < nk) {
        const T* kr = sm.kt[stage] + j * D;
        acc = 0.f;
        // rotated start so that lanes of a warp hit different banks
#pragma unroll 4
        for (int t = 0; t < D; ++t) {
          const int e = (t + j * 8) & (D - 1);
          acc = fmaf(sm.qs[h][e], to_f32(kr[e]), acc);
        }
        acc *= s.scale;
      }
      sm.p[h][j] = acc;
    }
    __syncthreads();
    for (int h = warp; h < G; h += kThreads / 32) {
      float m = -INFINITY;
      for (int j = lane; j < S; j += 32) m = fmaxf(m, sm.p[h][j]);
      m = warp_max(m);
      float l = 0.f;
      for (int j = lane; j < S; j += 32) {
        const float e = j < nk ? expf(sm.p[h][j] - m) : 0.f;
        sm.p[h][j] = e;
        l += e;
      }
      l = warp_sum(l);
      if (lane == 0) {
        sm.a[h] = sel ? s_sel[((long long)b * s.Hq + g * G + h) * s.K + slot] - logf(l) : m;
        sm.z[h] = l;
      }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < OUTS; ++r) {
      const int o = tid + r * kThreads;
      if (o < G * D) {
        const int h = o / D, e = o % D;
        float acc = 0.f;
        for (int j = 0; j < nk; ++j) acc = fmaf(sm.p[h][j], to_f32(sm.vt[stage][j * D + e]), acc);
        const float a = sm.a[h];
        const float Mn = fmaxf(Mh[h], a);
        const float cf = expf(Mh[h] - Mn), cu = expf(a - Mn);
        num[r] = num[r] * cf + cu * acc;
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float a = sm.a[h];
      const float Mn = fmaxf(Mh[h], a);
      den[h] = den[h] * expf(Mh[h] - Mn) + expf(a - Mn) * sm.z[h];
      Mh[h] = Mn;
    }
    __syncthreads();  // stage may now be refilled
  }
  if (!alive) {
    // a wait ran out: let copies this CTA issued land before its shared memory
    // is released (bounded as well), then leave the record undefined
    if (tid == 0)
      for (int st2 = 0; st2 < 2; ++st2)
        if (inflight[st2]) mbar_wait(&sm.full[st2], phase[st2], ctx);
    return;
  }
  // record: [B, Hq, nsplit, D + 2] = (M, den, num[D])
#pragma unroll
  for (int r = 0; r < OUTS; ++r) {
    const int o = tid + r * kThreads;
    if (o < G * D) {
      const int h = o / D, e = o % D;
      float* rec = ws + (((long long)b * s.Hq + g * G + h) * nsplit + split) * (D + 2);
      rec[2 + e] = num[r];
      if (e == 0) {
        rec[0] = Mh[h];
        rec[1] = den[h];
      }
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(D) attn_decode_merge(Shape s, const float* __restrict__ ws, T* __restrict__ out,
                                                       int nsplit) {
  const long long bh = blockIdx.x;
  const int e = threadIdx.x;
  const float* rec = ws + bh * nsplit * (D + 2);
  float M = -INFINITY;
  for (int x = 0; x < nsplit; ++x) M = fmaxf(M, rec[x * (D + 2)]);
  float num = 0.f, den = 0.f;
  for (int x = 0; x < nsplit; ++x) {
    const float m = rec[x * (D + 2)];
    if (m == -INFINITY) continue;
    const float w = expf(m - M);
    den += w * rec[x * (D + 2) + 1];
    num += w * rec[x * (D + 2) + 2 + e];
  }
  out[bh * D + e] = from_f32<T>(num / den);
}

// ---------------------------------------------------------------------------
// bf16, d = 128, S = 64: every warp gathers its tiles straight from HBM into
// tensor-core fragments (no shared-memory staging) and computes
//   S^T (64 keys x 8 cols) = K_tile . Q^T,   O^T (128 x 8 cols) += V_tile^T . P^T
// with the group's G <= 8 heads as the N = 8 columns (bf16 mma.sync, fp32
// accumulation); fragment layouts and line-wide loads: gather_mma.cuh.  Each warp folds its units with a running maximum
// per head; the CTA folds its warps in shared memory and writes one record
// per head, like the CUDA-core kernel above.  Registers are capped so that
// four CTAs fit on an SM, and the split count keeps the grid within four
// CTAs per SM: every CTA of a decode step is resident in one wave (measured
// faster than a grid of 2.2 waves at 186 registers, despite a few spills).
constexpr int kMmaWarps = 4;

template <int G>
__global__ void __launch_bounds__(kMmaWarps * 32, 4) attn_decode_mma(Shape s, const __nv_bfloat16* __restrict__ q,
                                                                  const __nv_bfloat16* __restrict__ k,
                                                                  const __nv_bfloat16* __restrict__ v,
                                                                  const int32_t* __restrict__ idx,
                                                                  const float* __restrict__ s_sel,
                                                                  float* __restrict__ ws, int nsplit, DecView dv, DevCtx ctx) {
  constexpr int D = 128, S = 64;
  __shared__ float red_acc[kMmaWarps][G][D];
  __shared__ float red_m[kMmaWarps][G], red_d[kMmaWarps][G];
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, c4 = lane & 3;
  int L = dv_len(dv, s, b);
  const bool len_ok = L >= 1 && L <= s.N;  // invalid: reported, no units (the record stays empty)
  if (!len_ok) {
    if (threadIdx.x == 0) raise_status(ctx, kStatusBadIndex);
    L = 1;
  }
  const int pos = L - 1, cur = pos / S;
  const int ncand = max(0, cur - s.nw + 1);
  const int wc0 = max(0, cur - s.nw + 1);
  const int nunits = len_ok ? s.K + (cur - wc0 + 1) : 0;
  const int32_t* ir = idx + ((long long)b * s.Hkv + g) * s.K;
  // Q^T as the B operand of S^T: column gq = head gq (zero past G)
  uint32_t qf[2][8];
  load_qcol(gq < G ? q + ((long long)b * s.Hq + g * G + gq) * D : nullptr, c4, qf);
  // this thread's columns 2c4, 2c4+1 (heads; >= G are padding)
  float acc[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  float M[2] = {-INFINITY, -INFINITY}, den[2] = {0.f, 0.f};

  // units of this CTA: u = split + nsplit * t; of this warp: every kMmaWarps-th of those
  for (int u = split + nsplit * warp; u < nunits; u += nsplit * kMmaWarps) {
    int nk;
    long long off;
    bool sel;
    int slot = -1;
    if (u < s.K) {
      const int c = ir[u];
      if (!list_entry_accepted(ir, u, ncand)) {  // the list form, common.cuh
        if (c != -1 && lane == 0) raise_status(ctx, kStatusBadIndex);
        continue;
      }
      sel = true;
      slot = u;
      off = dv_chunk(dv, s, b, g, c);
      nk = S;
    } else {
      sel = false;
      const int wc = wc0 + (u - s.K);
      off = dv_chunk(dv, s, b, g, wc);
      nk = min(S, L - wc * S);
    }
    if (off < 0) {  // a page outside the pool: reported, never read
      if (lane == 0) raise_status(ctx, kStatusBadIndex);
      continue;
    }
    const __nv_bfloat16* kc = k + off;
    const __nv_bfloat16* vc = v + off;
    const int kmax = nk - 1;
    float sc[4][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
    mma_st_tile(kc, kmax, gq, c4, qf, sc);
    // per column (head): m = max logit, l = sum e^{s-m}; log-weight lam
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int hcol = 2 * c4 + r;
      float mx = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          float t = sc[mt][2 * hi + r] * s.scale;
          if (16 * mt + gq + 8 * hi >= nk) t = -INFINITY;
          sc[mt][2 * hi + r] = t;
          mx = fmaxf(mx, t);
        }
      mx = col_max(mx);
      float l = 0.f;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const float t = sc[mt][2 * hi + r];
          const float p = t == -INFINITY ? 0.f : __expf(t - mx);
          sc[mt][2 * hi + r] = p;
          l += p;
        }
      l = col_sum(l);
      float lam = mx;
      if (sel && hcol < G) lam = __ldg(s_sel + ((long long)b * s.Hq + g * G + hcol) * s.K + slot) - __logf(l);
      if (hcol >= G) lam = -INFINITY;
      const float Mn = fmaxf(M[r], lam);
      if (Mn == -INFINITY) {
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) sc[mt][r] = sc[mt][2 + r] = 0.f;
        continue;
      }
      const float fo = __expf(M[r] - Mn), fu = __expf(lam - Mn);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        acc[mt][r] *= fo;
        acc[mt][2 + r] *= fo;
      }
      den[r] = den[r] * fo + fu * l;
      M[r] = Mn;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        sc[mt][r] *= fu;
        sc[mt][2 + r] *= fu;
      }
    }
    // O^T += V^T P^T
    mma_ot_tile(vc, kmax, gq, c4, sc, acc);
  }
  // fold the warps: thread holds dims 8 gq + mt and 64 + 8 gq + mt of columns 2c4, 2c4+1
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int hcol = 2 * c4 + r;
    if (hcol < G) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        red_acc[warp][hcol][8 * gq + mt] = acc[mt][r];
        red_acc[warp][hcol][64 + 8 * gq + mt] = acc[mt][2 + r];
      }
      if (gq == 0) {
        red_m[warp][hcol] = M[r];
        red_d[warp][hcol] = den[r];
      }
    }
  }
  __syncthreads();
  for (int o = threadIdx.x; o < G * D; o += kMmaWarps * 32) {
    const int h = o / D, e = o % D;
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kMmaWarps; ++w) Mx = fmaxf(Mx, red_m[w][h]);
    float num = 0.f, dd = 0.f;
#pragma unroll
    for (int w = 0; w < kMmaWarps; ++w) {
      if (red_m[w][h] == -INFINITY) continue;
      const float f = __expf(red_m[w][h] - Mx);
      num += f * red_acc[w][h][e];
      dd += f * red_d[w][h];
    }
    float* rec = ws + (((long long)b * s.Hq + g * G + h) * nsplit + split) * (D + 2);
    rec[2 + e] = num;
    if (e == 0) {
      rec[0] = Mx;
      rec[1] = dd;
    }
  }
}

template <int G>
cudaError_t go_mma(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                   const float* s_sel, void* out, void* ws, int nsplit, cudaStream_t st, const DevCtx& ctx,
                   const DecView& dv) {
  attn_decode_mma<G><<<dim3(nsplit, s.Hkv, s.B), kMmaWarps * 32, 0, st>>>(
      s, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, idx, s_sel, (float*)ws, nsplit,
      dv, ctx);
  attn_decode_merge<__nv_bfloat16, 128><<<s.B * s.Hq, 128, 0, st>>>(s, (const float*)ws, (__nv_bfloat16*)out,
                                                                     nsplit);
  return cudaGetLastError();
}

int pick_nsplit(const Shape& s) {
  const int cur = (s.N - 1) / s.S;
  const int nwin = cur - max(0, cur - s.nw + 1) + 1;
  const int nunits = s.K + nwin;
  const int sms = device_sm_count();
  const int groups = s.B * s.Hkv;
  int nsplit = (sms * 4) / groups;
  // one wave of four CTAs per SM; at most 16 units per CTA, at least one unit per CTA
  nsplit = max(nsplit, (nunits + 15) / 16);
  nsplit = min(nsplit, nunits);
  return max(nsplit, 1);
}

template <typename T, int D, int S, int G>
cudaError_t go(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx, const float* s_sel,
               void* out, void* ws, cudaStream_t st, const DevCtx& ctx, const DecView& dv) {
  const int nsplit = pick_nsplit(s);
  const size_t smem = sizeof(DecSmem<T, D, S, G>);
  auto kern = attn_decode_partial<T, D, S, G>;
  cudaError_t e = ensure_dynamic_smem((const void*)kern, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(nsplit, s.Hkv, s.B), kThreads, smem, st>>>(s, (const T*)q, (const T*)k, (const T*)v, idx, s_sel,
                                                         (float*)ws, nsplit, dv, ctx);
  attn_decode_merge<T, D><<<s.B * s.Hq, D, 0, st>>>(s, (const float*)ws, (T*)out, nsplit);
  return cudaGetLastError();
}

template <typename T, int D, int S>
cudaError_t go_g(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx, const float* s_sel,
                 void* out, void* ws, cudaStream_t st, const DevCtx& ctx, const DecView& dv) {
  switch (s.G) {
    case 1: return go<T, D, S, 1>(s, q, k, v, idx, s_sel, out, ws, st, ctx, dv);
    case 2: return go<T, D, S, 2>(s, q, k, v, idx, s_sel, out, ws, st, ctx, dv);
    case 4: return go<T, D, S, 4>(s, q, k, v, idx, s_sel, out, ws, st, ctx, dv);
    case 8: return go<T, D, S, 8>(s, q, k, v, idx, s_sel, out, ws, st, ctx, dv);
  }
  return cudaErrorNotSupported;
}

}  // namespace

// Fixed scratch for hils_attn_decode_noalloc: the split-KV partial records
// live here instead of in a caller-provided workspace.  Every GPU that loads
// the library holds this array until the process exits.
constexpr size_t kStaticScratchFloats = size_t(1) << 20;  // 4 MiB
static __device__ __align__(256) float g_decode_scratch[kStaticScratchFloats];

size_t decode_attn_workspace(const Shape& s) {
  const int nsplit = pick_nsplit(s);
  return (size_t)s.B * s.Hq * nsplit * (s.d + 2) * sizeof(float);
}

cudaError_t launch_attn_decode(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                               const float* s_sel, void* out, void* ws, cudaStream_t st, const DevCtx& ctx,
                               const DecView& dv) {
  if (s.dtype == 0) {
    if (s.d == 64 && s.S == 32) return go_g<float, 64, 32>(s, q, k, v, idx, s_sel, out, ws, st, ctx, dv);
    if (s.d == 64 && s.S == 64) return go_g<float, 64, 64>(s, q, k, v, idx, s_sel, out, ws, st, ctx, dv);
    if (s.d == 128 && s.S == 64) return go_g<float, 128, 64>(s, q, k, v, idx, s_sel, out, ws, st, ctx, dv);
    if (s.d == 128 && s.S == 32) return go_g<float, 128, 32>(s, q, k, v, idx, s_sel, out, ws, st, ctx, dv);
  } else if (s.d == 128 && s.S == 64) {
    const int nsplit = pick_nsplit(s);
    switch (s.G) {
      case 1: return go_mma<1>(s, q, k, v, idx, s_sel, out, ws, nsplit, st, ctx, dv);
      case 2: return go_mma<2>(s, q, k, v, idx, s_sel, out, ws, nsplit, st, ctx, dv);
      case 4: return go_mma<4>(s, q, k, v, idx, s_sel, out, ws, nsplit, st, ctx, dv);
      case 8: return go_mma<8>(s, q, k, v, idx, s_sel, out, ws, nsplit, st, ctx, dv);
    }
  }
  return cudaErrorNotSupported;
}

size_t decode_static_scratch_bytes() { return kStaticScratchFloats * sizeof(float); }

// Host code cannot pass g_decode_scratch itself (its host-side name is a
// stand-in, not a device address).  The device address is looked up once per
// device, with that device current, and cached.
cudaError_t launch_attn_decode_static(const Shape& s, const void* q, const void* k, const void* v,
                                      const int32_t* idx, const float* s_sel, void* out, cudaStream_t st,
                                      const DevCtx& ctx) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_decode_scratch);
      if (e != cudaSuccess) return e;
      addr[dev] = p;
    }
    ws = addr[dev];
  }
  return launch_attn_decode(s, q, k, v, idx, s_sel, out, ws, st, ctx, DecView{});
}

}  // namespace hils
