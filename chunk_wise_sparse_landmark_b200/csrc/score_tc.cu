// Chunk scoring + GQA group max + top-K on the tcgen05 tensor cores
// (bf16 prefill, d = 128, G = 4, K <= 64).
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method): surrogate score s^_{h,i,c} = q~_{h,i}.k'_{h,c} / sqrt(d) + b'_{h,c};
// third practical design choice: per-head scores, max over the heads of the
// GQA group, top-K chunks from the group score; candidates are the complete
// chunks before the chunk-aligned window.  The routing cost is O(N/S) per
// position (same section), i.e. a causal GEMM Q~ (N x d) . K'^T (d x N/S).
//
// One CTA = 128 positions (the MMA's M) of one (sequence, KV group).  The
// four heads' query tiles are written once into tensor memory and used as the
// A operand of every MMA (256 TMEM columns); k' tiles of 32 chunks x 128 for
// the four heads (32 KB) stream through a 3-stage TMA ring (128-byte swizzle,
// chunks past C read as zero); the 4 x 32 fp32 accumulators are
// double-buffered in tensor memory (256 columns).  Warp roles: 0 = TMA
// producer, 1 = MMA issuer (and TMEM owner), 2..5 = epilogue, one thread per
// position (its TMEM lane).
//
// Selection is exact and deterministic.  Pass 1 streams every tile and keeps,
// per row, the K largest keys key = (ordered bits of g) << 32 | (~c) (larger g
// first, ties to the smaller c): candidates above the current threshold are
// appended to a per-row buffer and folded into a min-heap of size K when any
// row of the warp could overflow.  Pass 2 recomputes the same tiles (same
// instructions, bit-identical scores) and emits every candidate whose key is
// >= the row's K-th key, in ascending chunk order, with each head's own s^.
#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int D = 128, G = 4;
constexpr int MQ = 128;   // positions per CTA
constexpr int TCH = 32;   // chunks per tile (MMA N)
constexpr int NSTB = 3;   // k' ring stages
constexpr int KMAX = 64;
constexpr int CAP = KMAX + TCH;
constexpr int THREADS = 192;
constexpr uint32_t BBOX = TCH * 128;          // one [32 chunks x 64 d] bf16 box
constexpr uint32_t BSTAGE = G * 2 * BBOX;     // 32 KB
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACOL = 0;                  // A: head h at ACOL + 64 h
constexpr uint32_t DCOL = 256;                // D stage sd, head h at DCOL + 128 sd + 32 h

struct __align__(1024) SmemS {
  unsigned char b[NSTB][G][2][BBOX];
  unsigned long long buf[CAP][MQ];  // column per row: conflict-free per-thread access
  alignas(16) float bt[2][G][TCH];  // b' of the tile in each accumulator stage
  uint64_t bfull[NSTB], bempty[NSTB], dfull[2], dempty[2], afull, done;
  uint32_t tmem;
};

HILS_DI unsigned long long make_key(float g, int c) {
  return ((unsigned long long)float_key(g) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)c);
}

// min-heap of K keys stored in column r of buf
HILS_DI void sift_down(SmemS& sm, int r, int K, int i, unsigned long long key) {
  while (true) {
    const int l = 2 * i + 1;
    if (l >= K) break;
    int m = l;
    if (l + 1 < K && sm.buf[l + 1][r] < sm.buf[l][r]) m = l + 1;
    if (sm.buf[m][r] >= key) break;
    sm.buf[i][r] = sm.buf[m][r];
    i = m;
  }
  sm.buf[i][r] = key;
}

__global__ void __launch_bounds__(THREADS, 1)
    score_topk_tc_kernel(Shape s, const __grid_constant__ CUtensorMap tmk, const __nv_bfloat16* __restrict__ q,
                         const float* __restrict__ b_sum, int32_t* __restrict__ idx, float* __restrict__ s_sel,
                         DevCtx ctx) {
  extern __shared__ unsigned char smem_raw[];
  SmemS& sm = *reinterpret_cast<SmemS*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y, b = blockIdx.z;
  const int i0 = blockIdx.x * MQ;
  const int K = s.K;
  const int last = min(i0 + MQ, s.N) - 1;
  const int ncand_max = max(0, last / 64 - s.nw + 1);
  const int T = (ncand_max + TCH - 1) / TCH;  // tiles per pass
  const int NIT = 2 * T;

  if (tid == 0) {
    for (int x = 0; x < NSTB; ++x) {
      mbar_init(&sm.bfull[x], 1);
      mbar_init(&sm.bempty[x], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.dfull[x], 1);
      mbar_init(&sm.dempty[x], 4);
    }
    mbar_init(&sm.afull, 4);
    mbar_init(&sm.done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;

  if (warp == 0) {
    // ---------------------------------------------------------- producer ----
    int last_round[NSTB] = {-1, -1, -1};
    if (lane == 0 && NIT > 0) prefetch_tmap(&tmk);
    bool ok = true;
    for (int it = 0; it < NIT && ok; ++it) {
      const int t = it % T, sb = it % NSTB, rnd = it / NSTB;
      if (rnd > 0) ok = mbar_wait(&sm.bempty[sb], (rnd - 1) & 1, ctx);
      if (!ok) break;
      if (lane == 0 && ctx.inject != 1) {
        mbar_arrive_expect_tx(&sm.bfull[sb], BSTAGE);
        for (int h = 0; h < G; ++h) {
          const int z = b * s.Hq + g * G + h;
          tma_load_3d(sm.b[sb][h][0], &tmk, 0, t * TCH, z, &sm.bfull[sb]);
          tma_load_3d(sm.b[sb][h][1], &tmk, 64, t * TCH, z, &sm.bfull[sb]);
        }
        last_round[sb] = rnd;
      }
      __syncwarp();
    }
    if (lane == 0)
      for (int x = 0; x < NSTB; ++x)
        if (last_round[x] >= 0) mbar_wait(&sm.bfull[x], last_round[x] & 1, ctx);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA ------
    const uint32_t idesc = idesc_bf16_f32(MQ, TCH);
    bool ok = NIT == 0 || mbar_wait(&sm.afull, 0, ctx);
    tc_fence_after();
    for (int it = 0; it < NIT && ok; ++it) {
      const int sb = it % NSTB, sd = it % 2;
      ok = mbar_wait(&sm.bfull[sb], (it / NSTB) & 1, ctx);
      if (ok && it >= 2) ok = mbar_wait(&sm.dempty[sd], ((it / 2) - 1) & 1, ctx);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t bdesc_addr = smem_u32(sm.b[sb][h][kk >> 2]) + (kk & 3) * 32;
            mma_ts(tmem + DCOL + sd * 128 + h * 32, tmem + ACOL + h * 64 + kk * 8, sdesc_k_sw128(bdesc_addr),
                   idesc, kk > 0 ? 1u : 0u);
          }
        }
        tc_commit(&sm.bempty[sb]);
        tc_commit(&sm.dfull[sd]);
      }
      __syncwarp();
    }
    // every MMA issued above has completed before the columns are released
    if (lane == 0) {
      tc_commit(&sm.done);
      mbar_wait(&sm.done, 0, ctx);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue ----
    const int qd = warp & 3;          // TMEM lane quadrant of this warp
    const int r = qd * 32 + lane;     // row = TMEM lane
    const int i = i0 + r;
    const bool valid = i < s.N;
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    // A: this row's scoring query for the four heads -> TMEM
    for (int h = 0; h < G; ++h) {
      const uint4* src = reinterpret_cast<const uint4*>(q + (((long long)b * s.Hq + g * G + h) * s.N + (valid ? i : 0)) * D);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t w[32];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const uint4 u = valid ? src[half * 8 + x] : make_uint4(0, 0, 0, 0);
          w[4 * x] = u.x;
          w[4 * x + 1] = u.y;
          w[4 * x + 2] = u.z;
          w[4 * x + 3] = u.w;
        }
        tmem_st32(lane_addr + ACOL + h * 64 + half * 32, w);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.afull);

    const int ncand = valid ? max(0, i / 64 - s.nw + 1) : 0;
    const float scale = s.scale;
    unsigned long long tau = 0ull;  // keys must exceed tau to enter
    int cnt = 0;
    bool heap = false;
    int nsel = 0;
    const long long row_idx = (((long long)b * s.Hkv + g) * s.N + i) * K;
    bool ok = true;

    auto fold = [&]() {  // fold buffered entries K..cnt-1 into the heap (this row)
      if (!heap) {
        if (cnt < K) return;
        for (int x = K / 2 - 1; x >= 0; --x) sift_down(sm, r, K, x, sm.buf[x][r]);
        heap = true;
      }
      for (int e = K; e < cnt; ++e) {
        const unsigned long long key = sm.buf[e][r];
        if (key > sm.buf[0][r]) sift_down(sm, r, K, 0, key);
      }
      cnt = K;
      tau = sm.buf[0][r];
    };

    for (int it = 0; it < NIT; ++it) {
      const int pass = it / T, t = it % T, sd = it % 2;
      const int c0 = t * TCH;
      const bool landed = mbar_wait(&sm.dfull[sd], (it / 2) & 1, ctx);
      if (!__all_sync(0xffffffffu, landed)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // b' of this tile, 4 heads x 32 chunks: one coalesced element per epilogue
      // thread into shared memory, then a barrier among the four epilogue warps
      {
        const int hh = r >> 5, jj = r & 31, cc = c0 + jj;
        sm.bt[sd][hh][jj] = cc < s.C ? __ldg(b_sum + ((long long)b * s.Hq + g * G + hh) * s.C + cc) : 0.f;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      // group score g = max_h (acc * scale + b'); identical in both passes
      uint32_t v[G][32];
#pragma unroll
      for (int h = 0; h < G; ++h) tmem_ld32(lane_addr + DCOL + sd * 128 + h * 32, v[h]);
      tmem_wait_ld();
      float gv[TCH];
#pragma unroll
      for (int j = 0; j < TCH; ++j) gv[j] = -INFINITY;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float4* bt4 = reinterpret_cast<const float4*>(sm.bt[sd][h]);
#pragma unroll
        for (int j4 = 0; j4 < TCH / 4; ++j4) {
          const float4 bb = bt4[j4];
          gv[4 * j4 + 0] = fmaxf(gv[4 * j4 + 0], __fmaf_rn(__uint_as_float(v[h][4 * j4 + 0]), scale, bb.x));
          gv[4 * j4 + 1] = fmaxf(gv[4 * j4 + 1], __fmaf_rn(__uint_as_float(v[h][4 * j4 + 1]), scale, bb.y));
          gv[4 * j4 + 2] = fmaxf(gv[4 * j4 + 2], __fmaf_rn(__uint_as_float(v[h][4 * j4 + 2]), scale, bb.z));
          gv[4 * j4 + 3] = fmaxf(gv[4 * j4 + 3], __fmaf_rn(__uint_as_float(v[h][4 * j4 + 3]), scale, bb.w));
        }
      }
      if (pass == 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.dempty[sd]);
#pragma unroll
        for (int j = 0; j < TCH; ++j) {
          const int c = c0 + j;
          if (c < ncand) {
            const unsigned long long key = make_key(gv[j], c);
            if (key > tau) sm.buf[cnt++][r] = key;
          }
        }
        if (__any_sync(0xffffffffu, cnt > CAP - TCH)) fold();
        if (t == T - 1) {
          fold();
          if (!heap) tau = 0ull;  // fewer than K candidates: take them all
          else tau = tau - 1ull;  // pass 2 takes keys >= the K-th key
        }
      } else {
        uint32_t selmask = 0;
#pragma unroll
        for (int j = 0; j < TCH; ++j) {
          const int c = c0 + j;
          if (c < ncand && make_key(gv[j], c) > tau) selmask |= 1u << j;
        }
        if (selmask != 0) {
          const int base = nsel;
#pragma unroll
          for (int j = 0; j < TCH; ++j) {
            if ((selmask >> j) & 1u) {
              const int slot = base + __popc(selmask & ((1u << j) - 1u));
              if (slot < K) {
                idx[row_idx + slot] = c0 + j;
#pragma unroll
                for (int h = 0; h < G; ++h)
                  s_sel[(((long long)b * s.Hq + g * G + h) * s.N + i) * K + slot] =
                      __fmaf_rn(__uint_as_float(v[h][j]), scale, sm.bt[sd][h][j]);
              }
            }
          }
          nsel = base + __popc(selmask);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.dempty[sd]);
      }
    }
    if (valid && ok) {
      if (nsel != min(ncand, K)) raise_status(ctx, kStatusBadIndex);
      nsel = min(nsel, K);
      for (int x = nsel; x < K; ++x) {
        idx[row_idx + x] = -1;
#pragma unroll
        for (int h = 0; h < G; ++h) s_sel[(((long long)b * s.Hq + g * G + h) * s.N + i) * K + x] = -INFINITY;
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

size_t score_tc_workspace(const Shape&) { return 0; }

cudaError_t launch_score_topk_tc(const Shape& s, const void* q, const void* k_sum, const float* b_sum, int32_t* idx,
                                 float* s_sel, cudaStream_t st, const DevCtx& ctx) {
  if (s.d != D || s.G != G || s.K > KMAX || s.S != 64) return cudaErrorNotSupported;
  CUtensorMap tmk;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)(s.C > 0 ? s.C : 1), (uint64_t)s.B * s.Hq};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)(s.C > 0 ? s.C : 1) * D * 2};
  const uint32_t box[3] = {64, TCH, 1};
  cudaError_t e = make_tmap_bf16(&tmk, k_sum, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(SmemS) + 1024;
  e = ensure_dynamic_smem((const void*)score_topk_tc_kernel, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((s.N + MQ - 1) / MQ, s.Hkv, s.B);
  score_topk_tc_kernel<<<grid, THREADS, smem, st>>>(s, tmk, (const __nv_bfloat16*)q, b_sum, idx, s_sel, ctx);
  return cudaGetLastError();
}

}  // namespace hils
