// Hierarchical-softmax sparse attention, bf16 prefill (d = 128, S = 64, G = 4).
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method): each selected chunk is attended with its own softmax, the chunk
// outputs are weighted by exp(s^_{i,c}) / Z^_i and the chunk-aligned window by
// Z_swa / Z^_i, Z^_i = sum_c exp(s^_{i,c}) + Z_swa.  The section's hardware
// paragraph attends the union of the chunks of a block of adjacent queries so
// that a loaded key/value tile serves every query of the block that chose it.
//
// One CTA = one query chunk: 64 positions x 4 heads = 256 rows of one
// (sequence, KV group).  Their fp32 output accumulators live in shared
// memory.  Phase A (selected chunks): a builder warp merges the 64 ascending
// chunk lists into a stream of (chunk, 64-bit position mask) items; every warp
// claims items dynamically, gathers the item's 64x128 key and value tiles
// once from L2 straight into tensor-core fragments, and computes the
// positions that chose the chunk two at a time (8 rows = the MMA's N):
// S^T = K Q^T, own-chunk softmax, weight e^{s^ - m_sel}/Z, O^T += V^T P^T,
// added into the shared accumulator rows (shared-memory atomics, since two
// items may touch the same row).  m_sel = max of the row's s^, fixed before
// the phase, so no rescaling is ever needed.  Phase B (window): each warp owns
// position pairs, runs the window chunks with an online softmax in registers,
// merges with the row's selected part, normalises and writes the output.
// Fragment layouts: gather_mma.cuh.  bf16 mma.sync, fp32 accumulation.
#include <climits>

#include "gather_mma.cuh"
#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int D = 128, S = 64, G = 4;
constexpr int P = 64;               // positions per CTA = one query chunk
constexpr int ROWS = P * G;         // 256
constexpr int NW = 16;              // warps
constexpr int THREADS = NW * 32;
constexpr int KMAX = 64;
constexpr int ACC_LD = ROWS + 1;    // pitch of acc[d][row]

struct SmemB {
  float acc[D][ACC_LD];
  float den[ROWS];                  // sum of e^{s^ - m_sel} over the row's chunks
  float msel[ROWS];                 // m_sel (log2 units), -inf without chunks
  int list[P][KMAX];                // (chunk << 8 | slot), ascending, INT_MAX past the end
  int item_c[P * KMAX];
  unsigned long long item_mask[P * KMAX];
  int published, next_item, total;
};

HILS_DI int chunk_of(int packed) { return packed == INT_MAX ? INT_MAX : (packed >> 8); }

__global__ void __launch_bounds__(THREADS, 1)
    attn_block_kernel(Shape s, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                      const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ idx,
                      const float* __restrict__ s_sel, __nv_bfloat16* __restrict__ out, DevCtx ctx) {
  extern __shared__ unsigned char smem_raw[];
  SmemB& sm = *reinterpret_cast<SmemB*>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, c4 = lane & 3;
  const int g = blockIdx.y, b = blockIdx.z;
  const int i0 = blockIdx.x * P;
  const int nq = min(P, s.N - i0);
  const int K = s.K;
  const int cur = i0 / S;
  const int ncand = max(0, cur - s.nw + 1);
  const long long kvbase = ((long long)b * s.Hkv + g) * (long long)s.N * D;
  const float sl2 = s.scale * kLog2e;

  // ------------------------------------------------------------- setup -----
  {
    float* a = &sm.acc[0][0];
    for (int e = tid; e < D * ACC_LD; e += THREADS) a[e] = 0.f;
  }
  for (int r = tid; r < ROWS; r += THREADS) {
    const int pl = r >> 2, h = r & 3;
    float mx = -INFINITY;
    if (pl < nq) {
      const float* sr = s_sel + (((long long)b * s.Hq + g * G + h) * s.N + i0 + pl) * K;
      for (int x = 0; x < K; ++x) mx = fmaxf(mx, __ldg(sr + x));
    }
    sm.msel[r] = mx * kLog2e;
    sm.den[r] = 0.f;
  }
  if (tid < P) {
    int n = 0;
    if (tid < nq) {
      const int32_t* ir = idx + (((long long)b * s.Hkv + g) * s.N + i0 + tid) * K;
      int prev = -1;
      for (int x = 0; x < K; ++x) {
        const int c = __ldg(ir + x);
        if (c < 0) continue;
        if (c >= ncand || c <= prev) {
          raise_status(ctx, kStatusBadIndex);
          continue;
        }
        sm.list[tid][n++] = (c << 8) | x;
        prev = c;
      }
    }
    for (; n < KMAX; ++n) sm.list[tid][n] = INT_MAX;
  }
  if (tid == 0) {
    sm.published = 0;
    sm.next_item = 0;
    sm.total = -1;
  }
  __syncthreads();

  // ------------------------------------------------ phase A: selected -----
  if (warp == NW - 1) {
    // builder: lane l merges positions l and l + 32
    int cu0 = 0, cu1 = 0, n = 0;
    const int* L0 = sm.list[lane];
    const int* L1 = sm.list[lane + 32];
    while (true) {
      const int v0 = cu0 < KMAX ? chunk_of(L0[cu0]) : INT_MAX;
      const int v1 = cu1 < KMAX ? chunk_of(L1[cu1]) : INT_MAX;
      const int c = __reduce_min_sync(0xffffffffu, min(v0, v1));
      if (c == INT_MAX) break;
      const unsigned m0 = __ballot_sync(0xffffffffu, v0 == c), m1 = __ballot_sync(0xffffffffu, v1 == c);
      cu0 += v0 == c;
      cu1 += v1 == c;
      if (lane == 0) {
        sm.item_c[n] = c;
        sm.item_mask[n] = (unsigned long long)m0 | ((unsigned long long)m1 << 32);
        __threadfence_block();
        *reinterpret_cast<volatile int*>(&sm.published) = n + 1;
      }
      ++n;
    }
    if (lane == 0) {
      __threadfence_block();
      *reinterpret_cast<volatile int*>(&sm.total) = n;
    }
    __syncwarp();
  }
  bool ok = true;
  while (true) {
    int it = 0;
    if (lane == 0) it = atomicAdd(&sm.next_item, 1);
    it = __shfl_sync(0xffffffffu, it, 0);
    // wait until the item is published or the stream has ended (bounded)
    bool have = false;
    if (lane == 0) {
      const long long t0 = clock64();
      while (true) {
        if (it < *reinterpret_cast<volatile int*>(&sm.published)) {
          have = true;
          break;
        }
        const int tot = *reinterpret_cast<volatile int*>(&sm.total);
        if (tot >= 0 && it >= tot) break;
        if (clock64() - t0 > ctx.wait_budget) {
          raise_status(ctx, kStatusTimeout);
          ok = false;
          break;
        }
        __nanosleep(64);
      }
      __threadfence_block();
    }
    have = __shfl_sync(0xffffffffu, have, 0);
    if (!have) break;
    const int c = sm.item_c[it];
    unsigned long long m = sm.item_mask[it];
    const __nv_bfloat16* kc = k + kvbase + (long long)c * S * D;
    const __nv_bfloat16* vc = v + kvbase + (long long)c * S * D;
    while (m) {
      const int pa = __ffsll((long long)m) - 1;
      m &= m - 1;
      int pb = -1;
      if (m) {
        pb = __ffsll((long long)m) - 1;
        m &= m - 1;
      }
      // columns: n < 4 -> (pa, head n), n >= 4 -> (pb, head n - 4)
      const int pcol = gq < 4 ? pa : pb;
      uint32_t qf[2][8];
      load_qcol(pcol >= 0 ? q + (((long long)b * s.Hq + g * G + (gq & 3)) * s.N + i0 + pcol) * D : nullptr, c4,
                qf);
      float sc[4][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
      mma_st_tile(kc, S - 1, gq, c4, qf, sc);
      const int mp = (c4 >> 1) ? pb : pa;  // this thread's position (columns 2c4, 2c4+1)
      const int mh = 2 * (c4 & 1);
      const bool mine = mp >= 0;
      float a2[2] = {-INFINITY, -INFINITY};
      if (mine) {
        const int* L = sm.list[mp];
        int lo = 0, hi = KMAX;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (chunk_of(L[mid]) < c) lo = mid + 1;
          else hi = mid;
        }
        const int slot = L[lo] & 255;
#pragma unroll
        for (int r = 0; r < 2; ++r)
          a2[r] = __ldg(s_sel + (((long long)b * s.Hq + g * G + mh + r) * s.N + i0 + mp) * K + slot) * kLog2e;
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float mx = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          sc[mt][r] *= sl2;
          sc[mt][2 + r] *= sl2;
          mx = fmaxf(mx, fmaxf(sc[mt][r], sc[mt][2 + r]));
        }
        mx = col_max(mx);
        float z = 0.f;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          sc[mt][r] = exp2f(sc[mt][r] - mx);
          sc[mt][2 + r] = exp2f(sc[mt][2 + r] - mx);
          z += sc[mt][r] + sc[mt][2 + r];
        }
        z = col_sum(z);
        const int row = mp * 4 + mh + r;
        float f = 0.f;
        if (mine) {
          const float w = exp2f(a2[r] - sm.msel[row]);  // <= 1
          f = w / z;
          if (gq == 0) atomicAdd(&sm.den[row], w);
        }
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          sc[mt][r] *= f;
          sc[mt][2 + r] *= f;
        }
      }
      float o[8][4];
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
      mma_ot_tile(vc, S - 1, gq, c4, sc, o);
      if (mine) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int row = mp * 4 + mh + r;
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            atomicAdd(&sm.acc[8 * gq + mt][row], o[mt][r]);
            atomicAdd(&sm.acc[64 + 8 * gq + mt][row], o[mt][2 + r]);
          }
        }
      }
    }
  }
  __syncthreads();

  // ------------------------------------------ phase B: window + output -----
  const int wc0 = max(0, cur - s.nw + 1);
  for (int pp = warp; pp < P / 2; pp += NW) {
    const int pa = 2 * pp, pb = 2 * pp + 1;
    if (pa >= nq) break;
    const bool vb = pb < nq;
    const int pcol = gq < 4 ? pa : pb;
    uint32_t qf[2][8];
    load_qcol((gq < 4 || vb) ? q + (((long long)b * s.Hq + g * G + (gq & 3)) * s.N + i0 + pcol) * D : nullptr, c4,
              qf);
    const int mp = (c4 >> 1) ? pb : pa;
    const int mh = 2 * (c4 & 1);
    const bool mine = (c4 >> 1) == 0 || vb;
    const int mypos = i0 + mp;
    float mw[2] = {-INFINITY, -INFINITY}, dw[2] = {0.f, 0.f};
    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    for (int wc = wc0; wc <= cur; ++wc) {
      const __nv_bfloat16* kc = k + kvbase + (long long)wc * S * D;
      const __nv_bfloat16* vcw = v + kvbase + (long long)wc * S * D;
      const int kmax = min(S - 1, s.N - 1 - wc * S);
      float sc[4][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
      mma_st_tile(kc, kmax, gq, c4, qf, sc);
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float mx = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            float t = sc[mt][2 * hi + r] * sl2;
            if (!mine || wc * S + 16 * mt + gq + 8 * hi > mypos) t = -INFINITY;
            sc[mt][2 * hi + r] = t;
            mx = fmaxf(mx, t);
          }
        mx = col_max(mx);
        if (mx > mw[r]) {
          const float f = exp2f(mw[r] - mx);
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            acc[mt][r] *= f;
            acc[mt][2 + r] *= f;
          }
          dw[r] *= f;
          mw[r] = mx;
        }
        float z = 0.f;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const float t = sc[mt][2 * hi + r];
            const float p = t == -INFINITY ? 0.f : exp2f(t - mw[r]);
            sc[mt][2 * hi + r] = p;
            z += p;
          }
        dw[r] += col_sum(z);
      }
      mma_ot_tile(vcw, kmax, gq, c4, sc, acc);
    }
    if (mine) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = mp * 4 + mh + r;
        const float ms = sm.msel[row];
        const float M = fmaxf(ms, mw[r]);
        const float fs = ms == -INFINITY ? 0.f : exp2f(ms - M);
        const float fw = exp2f(mw[r] - M);
        const float inv = 1.f / (sm.den[row] * fs + dw[r] * fw);
        float o[16];
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          o[mt] = (sm.acc[8 * gq + mt][row] * fs + acc[mt][r] * fw) * inv;
          o[8 + mt] = (sm.acc[64 + 8 * gq + mt][row] * fs + acc[mt][2 + r] * fw) * inv;
        }
        __nv_bfloat16* dst = out + (((long long)b * s.Hq + g * G + mh + r) * s.N + mypos) * D;
        uint4 lo, hi;
        lo.x = pack_bf16x2(o[0], o[1]);
        lo.y = pack_bf16x2(o[2], o[3]);
        lo.z = pack_bf16x2(o[4], o[5]);
        lo.w = pack_bf16x2(o[6], o[7]);
        hi.x = pack_bf16x2(o[8], o[9]);
        hi.y = pack_bf16x2(o[10], o[11]);
        hi.z = pack_bf16x2(o[12], o[13]);
        hi.w = pack_bf16x2(o[14], o[15]);
        *reinterpret_cast<uint4*>(dst + 8 * gq) = lo;
        *reinterpret_cast<uint4*>(dst + 64 + 8 * gq) = hi;
      }
    }
  }
}

}  // namespace

cudaError_t launch_attn_prefill_tc(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                   const float* s_sel, void* out, cudaStream_t st, const DevCtx& ctx) {
  if (s.d != D || s.S != S || s.G != G || s.K > KMAX) return cudaErrorNotSupported;
  const size_t smem = sizeof(SmemB) + 16;
  cudaError_t e = ensure_dynamic_smem((const void*)attn_block_kernel, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((s.N + P - 1) / P, s.Hkv, s.B);
  attn_block_kernel<<<grid, THREADS, smem, st>>>(s, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                                 (const __nv_bfloat16*)v, idx, s_sel, (__nv_bfloat16*)out, ctx);
  return cudaGetLastError();
}

}  // namespace hils
