// Hierarchical-softmax sparse attention, bf16 prefill (d = 128, S = 64, G = 4).
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method): each selected chunk is attended with its own softmax, the chunk
// outputs are weighted by exp(s^_{i,c}) / Z^_i and the chunk-aligned window by
// Z_swa / Z^_i, Z^_i = sum_c exp(s^_{i,c}) + Z_swa.  The section's hardware
// paragraph groups adjacent queries and attends the union of their chunks;
// here a warp groups 2 adjacent positions (8 query-head rows of one GQA group)
// and walks the union of their two chunk lists.
//
// Why this shape.  On inputs whose adjacent positions pick unrelated chunks,
// a loaded 64-key chunk is used by about one position (4 rows).  Staging
// chunks in shared memory for a block of positions then buys almost no reuse
// but costs a shared-memory write and read per chunk and ties each ring slot
// up while one warp computes.  Instead every warp gathers its own chunks
// straight from L2 into tensor-core fragments with coalesced 16-byte loads:
//
//   S^T (64 keys x 8 rows)   = K_c (keys x d)  . Q^T (d x rows)
//   O^T (128 d x 8 rows)    += V_c^T (d x keys) . P^T (keys x rows)
//
// bf16 mma.sync m16n8k16, fp32 accumulation.  Keys are the MMA's M, so the
// 8 rows fill N = 8 with no padding when both positions chose the chunk.  The
// contraction index d of S^T is permuted (consistently for K and Q) so that a
// thread's sixteen elements of four k-steps are one 32-byte vector and each
// warp load covers whole 128-byte lines; the M index of O^T is permuted so
// that the value loads of a key row are one contiguous line as well; P^T
// reaches B-fragment layout by an in-register 8x8 transpose (movmatrix).
//
// Row state (per query-head row): m2 = reference exponent (log2 units, >= all
// exponents used so far), den = sum of weights, acc = weighted values.
// Selected chunk: P_j = e^{s_j - mu}/Z_c * e^{s^ - m}, den += e^{s^ - m}.
// Window chunk: P_j = e^{s_j - m}, den += sum_j P_j; m is raised (acc and den
// rescaled) when a window logit exceeds it.  out = acc / den.
#include <climits>

#include "gather_mma.cuh"
#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int D = 128, S = 64, G = 4;
constexpr int WARPS = 4;            // per CTA; 2 positions per warp
constexpr int THREADS = WARPS * 32;
constexpr int POS_PER_CTA = 2 * WARPS;

__global__ void __launch_bounds__(THREADS, 3)
    attn_warp_kernel(Shape s, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                     const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ idx,
                     const float* __restrict__ s_sel, __nv_bfloat16* __restrict__ out, DevCtx ctx) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, c4 = lane & 3;  // fragment coordinates
  const int g = blockIdx.y, b = blockIdx.z;
  const int p0 = blockIdx.x * POS_PER_CTA + warp * 2;  // the warp's two positions p0, p0 + 1
  if (p0 >= s.N) return;
  const int K = s.K;
  const int cur = p0 / S;  // both positions share their chunk (p0 is even)
  const int ncand = max(0, cur - s.nw + 1);
  const bool valid1 = p0 + 1 < s.N;
  const long long kvbase = ((long long)b * s.Hkv + g) * (long long)s.N * D;
  const __nv_bfloat16* kb = k + kvbase;
  const __nv_bfloat16* vb = v + kvbase;

  // rows of the warp: n = 0..7 -> position p0 + n/4, head n%4.
  // B operand of S^T: row gq; the thread's rows for S^T columns / O^T columns: 2*c4, 2*c4+1
  // d is permuted: for k-step ks = 4jj + t (jj = 0,1; t = 0..3) thread c holds
  // logical k {2c, 2c+1} at physical d 64jj + 16c + 4t + {0,1} and {2c+8, 2c+9}
  // at 64jj + 16c + 4t + {2,3}, so one 32-byte load feeds four k-steps
  uint32_t qf[2][8];
  {
    const bool ok = (gq >> 2) == 0 || valid1;
    load_qcol(ok ? q + (((long long)b * s.Hq + g * G + (gq & 3)) * s.N + p0 + (gq >> 2)) * D : nullptr, c4, qf);
  }
  // this thread's two rows (columns of S^T / O^T): position my_q, heads my_h, my_h + 1
  const int my_q = c4 >> 1;  // 0 or 1
  const int my_h = 2 * (c4 & 1);
  const int my_pos = p0 + my_q;
  const bool my_valid = my_q == 0 || valid1;

  float acc[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  float m2[2], den[2] = {0.f, 0.f};
  // chunk lists of the two positions (broadcast loads, every lane walks both)
  const int32_t* L0 = idx + (((long long)b * s.Hkv + g) * s.N + p0) * K;
  const int32_t* L1 = L0 + K;
  const float* ss[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) ss[r] = s_sel + (((long long)b * s.Hq + g * G + my_h + r) * s.N + my_pos) * K;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float mx = -INFINITY;
    if (my_valid)
      for (int x = 0; x < K; ++x) mx = fmaxf(mx, __ldg(ss[r] + x));
    m2[r] = mx * kLog2e;
  }
  const float sl2 = s.scale * kLog2e;
  const int wc0 = max(0, cur - s.nw + 1);
  int cu0 = 0, cu1 = 0;  // cursors into L0, L1
  const int len1 = valid1 ? K : 0;
  auto head = [&](const int32_t* Lx, int& cu, int len) -> int {
    while (cu < len) {
      const int c = __ldg(Lx + cu);
      if (c >= 0 && c < ncand) return c;
      if (c >= ncand) raise_status(ctx, kStatusBadIndex);
      ++cu;  // skip -1 padding and invalid entries
    }
    return INT_MAX;
  };

  for (int step = 0;; ++step) {
    int c, slot_me = -1;
    bool win, part0, part1;
    if (step <= cur - wc0) {
      c = wc0 + step;
      win = true;
      part0 = true;
      part1 = valid1;
    } else {
      const int a0 = head(L0, cu0, K), a1 = head(L1, cu1, len1);
      c = min(a0, a1);
      if (c == INT_MAX) break;
      win = false;
      part0 = a0 == c;
      part1 = a1 == c;
      if (my_q == 0 && part0) slot_me = cu0;
      if (my_q == 1 && part1) slot_me = cu1;
      if (part0) ++cu0;
      if (part1) ++cu1;
    }
    const bool my_part = my_valid && (my_q == 0 ? part0 : part1);
    float a2[2] = {-INFINITY, -INFINITY};
    if (!win && my_part) {
      a2[0] = __ldg(ss[0] + slot_me) * kLog2e;
      a2[1] = __ldg(ss[1] + slot_me) * kLog2e;
    }
    const __nv_bfloat16* kc = kb + (long long)c * S * D;
    const __nv_bfloat16* vc = vb + (long long)c * S * D;
    // the current chunk may end past the sequence: clamp key rows to the last
    // valid one (those keys are causally masked, the load must stay in bounds)
    const int kmax = min(S - 1, s.N - 1 - c * S);

    // ---- S^T = K_c Q^T : 4 m-tiles (16 keys) x 8 k-steps (16 d)
    float sc[4][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
    mma_st_tile(kc, kmax, gq, c4, qf, sc);
    // ---- per-row weights; this thread holds keys 16mt+gq (+8) of rows 2c4, 2c4+1
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const int key = 16 * mt + gq + 8 * hi;
          float t = sc[mt][2 * hi + r] * sl2;
          if (!my_part || (win && c * S + key > my_pos)) t = -INFINITY;
          sc[mt][2 * hi + r] = t;
          mx = fmaxf(mx, t);
        }
      mx = col_max(mx);
      float base = mx;
      if (my_part && win && mx > m2[r]) {
        const float f = exp2f(m2[r] - mx);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          acc[mt][r] *= f;
          acc[mt][2 + r] *= f;
        }
        den[r] *= f;
        m2[r] = mx;
      }
      if (win) base = m2[r];
      float z = 0.f;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const float t = sc[mt][2 * hi + r];
          const float p = (my_part && t != -INFINITY) ? exp2f(t - base) : 0.f;
          sc[mt][2 * hi + r] = p;
          z += p;
        }
      z = col_sum(z);
      if (my_part) {
        if (win) {
          den[r] += z;
        } else {
          const float wgt = exp2f(a2[r] - m2[r]);  // <= 1
          den[r] += wgt;
          const float f = wgt / z;
#pragma unroll
          for (int mt = 0; mt < 4; ++mt) {
            sc[mt][r] *= f;
            sc[mt][2 + r] *= f;
          }
        }
      }
    }
    // ---- O^T += V_c^T P^T : 8 m-tiles (16 d) x 4 k-steps (16 keys)
    mma_ot_tile(vc, kmax, gq, c4, sc, acc);
  }

  // epilogue: this thread's rows 2c4, 2c4+1 (position my_pos, heads my_h, my_h+1),
  // output dims d = 8 gq + mt <- acc[mt][r] and 64 + 8 gq + mt <- acc[mt][2 + r]
  if (my_valid) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float inv = 1.f / den[r];
      __nv_bfloat16* o = out + (((long long)b * s.Hq + g * G + my_h + r) * s.N + my_pos) * D;
      uint4 lo, hi;
      lo.x = pack_bf16x2(acc[0][r] * inv, acc[1][r] * inv);
      lo.y = pack_bf16x2(acc[2][r] * inv, acc[3][r] * inv);
      lo.z = pack_bf16x2(acc[4][r] * inv, acc[5][r] * inv);
      lo.w = pack_bf16x2(acc[6][r] * inv, acc[7][r] * inv);
      hi.x = pack_bf16x2(acc[0][2 + r] * inv, acc[1][2 + r] * inv);
      hi.y = pack_bf16x2(acc[2][2 + r] * inv, acc[3][2 + r] * inv);
      hi.z = pack_bf16x2(acc[4][2 + r] * inv, acc[5][2 + r] * inv);
      hi.w = pack_bf16x2(acc[6][2 + r] * inv, acc[7][2 + r] * inv);
      *reinterpret_cast<uint4*>(o + 8 * gq) = lo;
      *reinterpret_cast<uint4*>(o + 64 + 8 * gq) = hi;
    }
  }
}

}  // namespace

cudaError_t launch_attn_prefill_tc(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                   const float* s_sel, void* out, cudaStream_t st, const DevCtx& ctx) {
  if (s.d != D || s.S != S || s.G != G || s.K > 64) return cudaErrorNotSupported;
  dim3 grid((s.N + POS_PER_CTA - 1) / POS_PER_CTA, s.Hkv, s.B);
  attn_warp_kernel<<<grid, THREADS, 0, st>>>(s, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                             (const __nv_bfloat16*)v, idx, s_sel, (__nv_bfloat16*)out, ctx);
  return cudaGetLastError();
}

}  // namespace hils
