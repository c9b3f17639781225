// Hierarchical-softmax sparse attention, bf16 prefill (d = 128, S = 64, G = 4).
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method): each selected chunk is attended with its own softmax, the chunk
// outputs are weighted by exp(s^_{i,c}) / Z^_i and the chunk-aligned window by
// Z_swa / Z^_i, Z^_i = sum_c exp(s^_{i,c}) + Z_swa.  The same section's
// hardware paragraph groups adjacent queries and attends the union of their
// chunks so that loaded key/value tiles are reused; that is the prior art this
// kernel keeps, adapted to what the reuse actually is.
//
// Design.  One CTA = 32 consecutive positions of one (sequence, KV group):
// 32 positions x 4 query heads = 128 rows.  A producer warp merges the 32
// ascending chunk lists into one ascending union stream (warp min + ballot per
// step), prepends the window chunks, and for every union chunk TMA-loads its
// 64x128 key and value tiles (128-byte swizzled boxes) into a 4-stage ring.
// Eight consumer warps each own 4 positions x 4 heads = one 16-row MMA tile
// with its accumulator in registers; a warp computes a chunk only if one of
// its positions selected it (or it is a window chunk), so every loaded tile
// is shared by all rows of the CTA that use it.  Scores and P.V run on the
// tensor cores (bf16 mma.sync, fp32 accumulation); the per-chunk softmax,
// the hierarchical weights and the window's online softmax are fp32.
//
// Row state: m2 = reference exponent (log2 domain, >= every exponent used so
// far), den = sum of weights, acc = weighted sum of values.  Selected chunk c:
// P_j = e^{s_j - mu} / Z_c * e^{s^_c - m}, den += e^{s^_c - m}.  Window chunk:
// P_j = e^{s_j - m}, den += sum_j P_j, with m raised (and acc, den rescaled)
// when a window logit exceeds it.  out = acc / den.
#include <climits>

#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int D = 128, S = 64, G = 4;
constexpr int QB = 32;  // positions per CTA
constexpr int NCW = 8;  // consumer warps (4 positions each)
constexpr int NST = 4;  // ring stages
constexpr int KMAX = 64;
constexpr int THREADS = (NCW + 1) * 32;
constexpr uint32_t BOX_BYTES = 64 * 64 * 2;        // 64 rows x 128 B
constexpr uint32_t STAGE_BYTES = 4 * BOX_BYTES;     // K (2 boxes) + V (2 boxes)

struct __align__(1024) Smem {
  __nv_bfloat16 kv[NST][4][64 * 64];  // [stage][K box0, K box1, V box0, V box1][64 rows x 64 cols]
  int idx[QB][KMAX];
  float ssel[QB][G][KMAX];
  int meta_c[NST];
  uint32_t meta_mask[NST];
  int meta_win[NST];
  uint64_t full[NST];
  uint64_t empty[NST];
};

// byte offset of (row, 16-byte chunk) inside a 64x128B box with 128B swizzle
HILS_DI uint32_t swz(int row, int chunk16) { return (uint32_t)(row * 128 + ((chunk16 ^ (row & 7)) << 4)); }

HILS_DI uint32_t ld_b32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

__global__ void __launch_bounds__(THREADS, 1)
    attn_union_kernel(Shape s, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                      const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ idx,
                      const float* __restrict__ s_sel, __nv_bfloat16* __restrict__ out, DevCtx ctx) {
  extern __shared__ unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y, b = blockIdx.z;
  const int i0 = blockIdx.x * QB;
  const int nq = min(QB, s.N - i0);
  const int K = s.K;
  const int cur = i0 / S;  // all 32 positions share their chunk (QB divides S)
  const int ncand = max(0, cur - s.nw + 1);

  // stage the block's chunk lists and surrogate scores; sanitise the lists
  for (int e = tid; e < QB * K; e += THREADS) {
    const int qi = e / K, x = e % K;
    int c = -1;
    if (qi < nq) {
      const int32_t* ir = idx + (((long long)b * s.Hkv + g) * s.N + i0 + qi) * K;
      c = ir[x];
      if (c >= ncand || (c >= 0 && x > 0 && ir[x - 1] >= c)) {
        raise_status(ctx, kStatusBadIndex);
        c = -1;
      }
    }
    sm.idx[qi][x] = c;
  }
  for (int e = tid; e < QB * G * K; e += THREADS) {
    const int qi = e / (G * K), h = (e / K) % G, x = e % K;
    sm.ssel[qi][h][x] =
        qi < nq ? s_sel[(((long long)b * s.Hq + g * G + h) * s.N + i0 + qi) * K + x] : -INFINITY;
  }
  if (tid == 0) {
    for (int st = 0; st < NST; ++st) {
      mbar_init(&sm.full[st], 1);
      mbar_init(&sm.empty[st], NCW);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == NCW) {
    // ------------------------------------------------------------ producer --
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
    int it = 0;
    int last_round[NST];
#pragma unroll
    for (int st = 0; st < NST; ++st) last_round[st] = -1;
    bool ok = true;
    const int zc = b * s.Hkv + g;
    auto emit = [&](int c, uint32_t mask, int win) {
      const int st = it % NST, round = it / NST;
      if (round > 0 && ok) ok = mbar_wait(&sm.empty[st], (round - 1) & 1, ctx);
      if (!ok) return;
      if (lane == 0) {
        sm.meta_c[st] = c;
        sm.meta_mask[st] = mask;
        sm.meta_win[st] = win;
        if (ctx.inject != 1) {
          if (c >= 0) {
            mbar_arrive_expect_tx(&sm.full[st], STAGE_BYTES);
            tma_load_3d(sm.kv[st][0], &tmk, 0, c * S, zc, &sm.full[st]);
            tma_load_3d(sm.kv[st][1], &tmk, 64, c * S, zc, &sm.full[st]);
            tma_load_3d(sm.kv[st][2], &tmv, 0, c * S, zc, &sm.full[st]);
            tma_load_3d(sm.kv[st][3], &tmv, 64, c * S, zc, &sm.full[st]);
            last_round[st] = round;
          } else {
            mbar_arrive(&sm.full[st]);
            last_round[st] = round;  // completes after (so implies) the stage's earlier phases
          }
        }
      }
      __syncwarp();
      ++it;
    };
    const int wc0 = max(0, cur - s.nw + 1);
    for (int wc = wc0; wc <= cur && ok; ++wc) emit(wc, 0xffffffffu, 1);
    int p = 0;
    const int* L = sm.idx[lane];
    while (ok) {
      while (p < K && L[p] < 0) ++p;
      const int v = p < K ? L[p] : INT_MAX;
      const int c = __reduce_min_sync(0xffffffffu, v);
      if (c == INT_MAX) break;
      const uint32_t mask = __ballot_sync(0xffffffffu, v == c);
      if (v == c) ++p;
      emit(c, mask, 0);
    }
    emit(-1, 0u, 0);
    // let every copy this CTA issued land before the CTA can retire (bounded)
    if (lane == 0)
      for (int st = 0; st < NST; ++st)
        if (last_round[st] >= 0) mbar_wait(&sm.full[st], last_round[st] & 1, ctx);
    return;
  }

  // -------------------------------------------------------------- consumers --
  const int gq = lane >> 2, c4 = lane & 3;
  const int h = gq & 3;
  const int qloc[2] = {warp * 4 + (gq >> 2), warp * 4 + (gq >> 2) + 2};
  bool valid[2];
  valid[0] = qloc[0] < nq;
  valid[1] = qloc[1] < nq;
  const int hq = g * G + h;
  const float sl2 = s.scale * kLog2e;

  // Q fragments (A operand, 16 rows x 128), rows gq and gq + 8
  uint32_t qf[8][4];
  {
    const __nv_bfloat16* q0 = q + (((long long)b * s.Hq + hq) * s.N + i0 + (valid[0] ? qloc[0] : 0)) * D;
    const __nv_bfloat16* q1 = q + (((long long)b * s.Hq + hq) * s.N + i0 + (valid[1] ? qloc[1] : 0)) * D;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int d0 = ks * 16 + 2 * c4;
      qf[ks][0] = valid[0] ? ld_b32(q0 + d0) : 0u;
      qf[ks][1] = valid[1] ? ld_b32(q1 + d0) : 0u;
      qf[ks][2] = valid[0] ? ld_b32(q0 + d0 + 8) : 0u;
      qf[ks][3] = valid[1] ? ld_b32(q1 + d0 + 8) : 0u;
    }
  }
  float acc[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  float m2[2], den[2];
  int cursor[2] = {0, 0};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float mx = -INFINITY;
    for (int x = 0; x < K; ++x) mx = fmaxf(mx, sm.ssel[qloc[r]][h][x]);
    m2[r] = mx * kLog2e;
    den[r] = 0.f;
  }
  const int pos[2] = {i0 + qloc[0], i0 + qloc[1]};

  for (int it = 0;; ++it) {
    const int st = it % NST;
    const bool landed = mbar_wait(&sm.full[st], (it / NST) & 1, ctx);
    if (!__all_sync(0xffffffffu, landed)) break;
    const int c = sm.meta_c[st];
    if (c < 0) break;
    const uint32_t mask = sm.meta_mask[st];
    const bool win = sm.meta_win[st] != 0;
    // participation and surrogate score per row
    bool part[2];
    float a2[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      part[r] = valid[r] && (win || ((mask >> qloc[r]) & 1u));
      a2[r] = -INFINITY;
      if (!win && part[r]) {
        const int* L = sm.idx[qloc[r]];
        while (cursor[r] < K && L[cursor[r]] < c) ++cursor[r];
        if (cursor[r] < K && L[cursor[r]] == c) {
          a2[r] = sm.ssel[qloc[r]][h][cursor[r]] * kLog2e;
        } else {
          part[r] = false;
        }
      }
    }
    if (__any_sync(0xffffffffu, part[0] || part[1])) {
      const uint32_t kbase = smem_u32(sm.kv[st][0]);
      const uint32_t vbase = smem_u32(sm.kv[st][2]);
      float sc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
      // S = Q K^T  (16 rows x 64 keys)
      {
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int dch = ks * 2 + (mi & 1);  // 16-byte chunk along d (0..15)
          const uint32_t box = kbase + (dch >> 3) * BOX_BYTES;
#pragma unroll
          for (int np = 0; np < 4; ++np) {
            const int key = np * 16 + (mi >> 1) * 8 + rr;
            uint32_t bf[4];
            ldmatrix_x4(bf, box + swz(key, dch & 7));
            mma_bf16_16816(sc[2 * np], qf[ks], bf[0], bf[1]);
            mma_bf16_16816(sc[2 * np + 1], qf[ks], bf[2], bf[3]);
          }
        }
      }
      // per-row weights (rows gq: elements 0,1; gq+8: elements 2,3)
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float mx = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = nt * 8 + 2 * c4 + e;
            float t = sc[nt][2 * r + e] * sl2;
            if (!part[r] || (win && c * S + key > pos[r])) t = -INFINITY;
            sc[nt][2 * r + e] = t;
            mx = fmaxf(mx, t);
          }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        float base, mul;
        if (!part[r]) {
          base = 0.f;
          mul = 0.f;
        } else if (win) {
          if (mx > m2[r]) {
            const float f = exp2f(m2[r] - mx);
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
              acc[nt][2 * r] *= f;
              acc[nt][2 * r + 1] *= f;
            }
            den[r] *= f;
            m2[r] = mx;
          }
          base = m2[r];
          mul = 1.f;
        } else {
          base = mx;
          mul = 1.f;  // scaled below once Z_c is known
        }
        float z = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float t = sc[nt][2 * r + e];
            const float p = (mul != 0.f && t != -INFINITY) ? exp2f(t - base) : 0.f;
            sc[nt][2 * r + e] = p;
            z += p;
          }
        z += __shfl_xor_sync(0xffffffffu, z, 1);
        z += __shfl_xor_sync(0xffffffffu, z, 2);
        if (part[r]) {
          if (win) {
            den[r] += z;
          } else {
            const float wgt = exp2f(a2[r] - m2[r]);  // <= 1: m2 >= every s^ of the row
            den[r] += wgt;
            const float f = wgt / z;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
              sc[nt][2 * r] *= f;
              sc[nt][2 * r + 1] *= f;
            }
          }
        }
      }
      // acc += P V   (16 rows x 128)
      {
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t pa[4];
          pa[0] = pack_bf16x2(sc[2 * kk][0], sc[2 * kk][1]);
          pa[1] = pack_bf16x2(sc[2 * kk][2], sc[2 * kk][3]);
          pa[2] = pack_bf16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
          pa[3] = pack_bf16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
          const int key = kk * 16 + (mi & 1) * 8 + rr;
#pragma unroll
          for (int np = 0; np < 8; ++np) {
            const int dch = np * 2 + (mi >> 1);
            uint32_t bf[4];
            ldmatrix_x4_trans(bf, vbase + (dch >> 3) * BOX_BYTES + swz(key, dch & 7));
            mma_bf16_16816(acc[2 * np], pa, bf[0], bf[1]);
            mma_bf16_16816(acc[2 * np + 1], pa, bf[2], bf[3]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[st]);
  }

  // epilogue: out = acc / den
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (!valid[r]) continue;
    const float inv = 1.f / den[r];
    __nv_bfloat16* o = out + (((long long)b * s.Hq + hq) * s.N + pos[r]) * D;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int d0 = nt * 8 + 2 * c4;
      *reinterpret_cast<uint32_t*>(o + d0) = pack_bf16x2(acc[nt][2 * r] * inv, acc[nt][2 * r + 1] * inv);
    }
  }
}

}  // namespace

cudaError_t launch_attn_prefill_tc(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                   const float* s_sel, void* out, cudaStream_t st, const DevCtx& ctx) {
  if (s.d != D || s.S != S || s.G != G || s.K > KMAX) return cudaErrorNotSupported;
  CUtensorMap tmk, tmv;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)s.N, (uint64_t)s.B * s.Hkv};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)s.N * D * 2};
  const uint32_t box[3] = {64, 64, 1};
  cudaError_t e = make_tmap_bf16(&tmk, k, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tmv, v, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(Smem) + 1024;
  e = ensure_dynamic_smem((const void*)attn_union_kernel, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((s.N + QB - 1) / QB, s.Hkv, s.B);
  attn_union_kernel<<<grid, THREADS, smem, st>>>(s, tmk, tmv, (const __nv_bfloat16*)q, idx, s_sel,
                                                 (__nv_bfloat16*)out, ctx);
  return cudaGetLastError();
}

}  // namespace hils
