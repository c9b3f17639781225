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
// the four heads (32 KB) stream through a 2-stage TMA ring (128-byte swizzle,
// chunks past C read as zero); the 4 x 32 fp32 accumulators are
// double-buffered in tensor memory (256 columns).  Warp roles: 0 = TMA
// producer, 1 = MMA issuer (and TMEM owner), 2..9 = epilogue: two threads per
// position (its TMEM lane), one per half of each 32-chunk tile.
//
// Selection is exact and deterministic.  Pass 1 streams every tile; each
// epilogue thread keeps the K largest keys of its half, key = (ordered bits of
// g) << 32 | (~c) (larger g first, ties to the smaller c): candidates above
// the current threshold go to a per-thread buffer of K + 16 entries that is
// folded into a min-heap of size K whenever it could overflow.  After the
// last tile the two halves of a row are merged, giving the row's K-th key.
// Pass 2 recomputes the same tiles (same instructions, bit-identical scores)
// and emits every candidate whose key is >= the K-th key, in ascending chunk
// order (the halves exchange their per-tile counts), with each head's own s^.
#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int D = 128, G = 4;
constexpr int MQ = 128;   // positions per CTA
constexpr int TCH = 32;   // chunks per tile (MMA N)
constexpr int HALF = TCH / 2;
constexpr int NSTB = 2;   // k' ring stages
constexpr int KMAX = 64;
constexpr int THREADS = 320;
constexpr int EPI = 256;  // epilogue threads
constexpr uint32_t BBOX = TCH * 128;          // one [32 chunks x 64 d] bf16 box
constexpr uint32_t BSTAGE = G * 2 * BBOX;     // 32 KB
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACOL = 0;                  // A: head h at ACOL + 64 h
constexpr uint32_t DCOL = 256;                // D stage sd, head h at DCOL + 128 sd + 32 h

// Fixed part of the shared memory; the per-thread key buffers follow it
// (K + 16 entries per thread, one column per thread).
struct __align__(1024) SmemS {
  unsigned char b[NSTB][G][2][BBOX];
  alignas(16) float bt[2][G][TCH];     // b' of the tile in each accumulator stage
  uint8_t cnt[2][MQ];                  // per-tile selection counts of each half (pass 2)
  uint64_t bfull[NSTB], bempty[NSTB], dfull[2], dempty[2], afull, done;
  uint32_t tmem;
};

HILS_DI unsigned long long make_key(float g, int c) {
  return ((unsigned long long)float_key(g) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)c);
}
// the float whose ordered image is the high word of `key` (-inf for key 0)
HILS_DI float key_float(unsigned long long key) {
  if (key == 0ull) return -INFINITY;
  const uint32_t u = (uint32_t)(key >> 32);
  return (u & 0x80000000u) ? __uint_as_float(u & 0x7FFFFFFFu) : __uint_as_float(~u);
}

// min-heap of K keys in column `col` of buf (pitch EPI)
HILS_DI void sift_down(unsigned long long* buf, int col, int K, int i, unsigned long long key) {
  while (true) {
    const int l = 2 * i + 1;
    if (l >= K) break;
    int m = l;
    if (l + 1 < K && buf[(l + 1) * EPI + col] < buf[l * EPI + col]) m = l + 1;
    if (buf[m * EPI + col] >= key) break;
    buf[i * EPI + col] = buf[m * EPI + col];
    i = m;
  }
  buf[i * EPI + col] = key;
}

struct TopK {
  int cnt = 0;
  bool heap = false;
  unsigned long long tau = 0ull;  // keys must exceed tau to enter
  float tau_f = -INFINITY;        // cheap pre-filter: g >= tau_f
};

// fold buffered entries K..cnt-1 into the heap (building it once cnt >= K)
HILS_DI void fold(unsigned long long* buf, int col, int K, TopK& t) {
  if (!t.heap) {
    if (t.cnt < K) return;
    for (int x = K / 2 - 1; x >= 0; --x) sift_down(buf, col, K, x, buf[x * EPI + col]);
    t.heap = true;
  }
  for (int e = K; e < t.cnt; ++e) {
    const unsigned long long key = buf[e * EPI + col];
    if (key > buf[col]) sift_down(buf, col, K, 0, key);
  }
  t.cnt = K;
  t.tau = buf[col];
  t.tau_f = key_float(t.tau);
}

HILS_DI void epi_barrier() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// barrier among the epilogue warps that also ANDs a flag, so that all of them
// take the same branch (nobody is left waiting at a later barrier)
HILS_DI bool epi_all(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)v)
      : "memory");
  return out != 0;
}

HILS_DI void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__global__ void __launch_bounds__(THREADS, 1)
    score_topk_tc_kernel(Shape s, const __grid_constant__ CUtensorMap tmk, const __nv_bfloat16* __restrict__ q,
                         const float* __restrict__ b_sum, int32_t* __restrict__ idx, float* __restrict__ s_sel,
                         DevCtx ctx) {
  extern __shared__ unsigned char smem_raw[];
  SmemS& sm = *reinterpret_cast<SmemS*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned long long* buf = reinterpret_cast<unsigned long long*>(&sm + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y, b = blockIdx.z;
  const int i0 = blockIdx.x * MQ;
  const int K = s.K;
  const int CAP = K + HALF;
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
      mbar_init(&sm.dempty[x], EPI / 32);
    }
    mbar_init(&sm.afull, EPI / 32);
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
    int last_round[NSTB];
#pragma unroll
    for (int x = 0; x < NSTB; ++x) last_round[x] = -1;
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
    const int e = warp - 2;           // 0..7
    const int hf = e >> 2;            // half of each tile: chunks [16 hf, 16 hf + 16)
    const int qd = warp & 3;          // TMEM lane quadrant of this warp
    const int r = qd * 32 + lane;     // row = TMEM lane
    const int col = hf * MQ + r;      // buffer column of this thread
    const int i = i0 + r;
    const bool valid = i < s.N;
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    // A: this row's scoring query, heads 2 hf and 2 hf + 1 -> TMEM
    for (int h = 2 * hf; h < 2 * hf + 2; ++h) {
      const uint4* src =
          reinterpret_cast<const uint4*>(q + (((long long)b * s.Hq + g * G + h) * s.N + (valid ? i : 0)) * D);
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
    TopK tk;
    int nsel = 0;
    const long long row_idx = (((long long)b * s.Hkv + g) * s.N + i) * K;
    bool ok = true;

    for (int it = 0; it < NIT; ++it) {
      const int pass = it / T, t = it % T, sd = it % 2;
      const int c0 = t * TCH + hf * HALF;  // first chunk of this thread's half
      const bool landed = mbar_wait(&sm.dfull[sd], (it / 2) & 1, ctx);
      if (!epi_all(landed)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (hf == 0) {
        const int hh = r >> 5, jj = r & 31, cc = t * TCH + jj;
        sm.bt[sd][hh][jj] = cc < s.C ? __ldg(b_sum + ((long long)b * s.Hq + g * G + hh) * s.C + cc) : 0.f;
      }
      epi_barrier();
      uint32_t v[G][HALF];
#pragma unroll
      for (int h = 0; h < G; ++h) tmem_ld16(lane_addr + DCOL + sd * 128 + h * 32 + hf * HALF, v[h]);
      tmem_wait_ld();
      float gv[HALF];
#pragma unroll
      for (int j = 0; j < HALF; ++j) gv[j] = -INFINITY;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float4* bt4 = reinterpret_cast<const float4*>(&sm.bt[sd][h][hf * HALF]);
#pragma unroll
        for (int j4 = 0; j4 < HALF / 4; ++j4) {
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
        for (int j = 0; j < HALF; ++j) {
          const int c = c0 + j;
          if (c < ncand && gv[j] >= tk.tau_f) {
            const unsigned long long key = make_key(gv[j], c);
            if (key > tk.tau) buf[(tk.cnt++) * EPI + col] = key;
          }
        }
        if (__any_sync(0xffffffffu, tk.heap ? tk.cnt > K : tk.cnt >= K)) fold(buf, col, K, tk);
        if (t == T - 1) {
          // merge the two halves of each row: half 1 hands its entries to half 0
          fold(buf, col, K, tk);
          if (hf == 1) sm.cnt[0][r] = (uint8_t)tk.cnt;
          epi_barrier();
          if (hf == 0) {
            const int n1 = sm.cnt[0][r];
            for (int x = 0; x < n1; ++x) {
              const unsigned long long key = buf[x * EPI + MQ + r];
              if (key > tk.tau) {
                buf[(tk.cnt++) * EPI + col] = key;
                if (tk.cnt == CAP || (!tk.heap && tk.cnt >= K)) fold(buf, col, K, tk);
              }
            }
            fold(buf, col, K, tk);
          }
          epi_barrier();  // half 1's entries have been read; its column is free
          if (hf == 0) buf[MQ + r] = tk.heap ? tk.tau - 1ull : 0ull;
          epi_barrier();
          // pass 2 takes keys >= the row's K-th key (all candidates if fewer than K)
          tk.tau = buf[MQ + r];
          tk.tau_f = key_float(tk.tau);
        }
      } else {
        uint32_t selmask = 0;
#pragma unroll
        for (int j = 0; j < HALF; ++j) {
          const int c = c0 + j;
          if (c < ncand && gv[j] >= tk.tau_f && make_key(gv[j], c) > tk.tau) selmask |= 1u << j;
        }
        sm.cnt[hf][r] = (uint8_t)__popc(selmask);
        epi_barrier();
        const int n0 = sm.cnt[0][r], n1 = sm.cnt[1][r];
        epi_barrier();  // counts consumed before the next tile overwrites them
        const int base = nsel + (hf ? n0 : 0);
        if (selmask != 0) {
#pragma unroll
          for (int j = 0; j < HALF; ++j) {
            if ((selmask >> j) & 1u) {
              const int slot = base + __popc(selmask & ((1u << j) - 1u));
              if (slot < K) {
                idx[row_idx + slot] = c0 + j;
#pragma unroll
                for (int h = 0; h < G; ++h)
                  s_sel[(((long long)b * s.Hq + g * G + h) * s.N + i) * K + slot] =
                      __fmaf_rn(__uint_as_float(v[h][j]), scale, sm.bt[sd][h][hf * HALF + j]);
              }
            }
          }
        }
        nsel += n0 + n1;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.dempty[sd]);
      }
    }
    if (valid && ok && hf == 0) {
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

size_t smem_bytes(int K) { return sizeof(SmemS) + 1024 + (size_t)(K + HALF) * EPI * sizeof(unsigned long long); }

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
  e = ensure_dynamic_smem((const void*)score_topk_tc_kernel, (int)smem_bytes(KMAX));
  if (e != cudaSuccess) return e;
  dim3 grid((s.N + MQ - 1) / MQ, s.Hkv, s.B);
  score_topk_tc_kernel<<<grid, THREADS, smem_bytes(s.K), st>>>(s, tmk, (const __nv_bfloat16*)q, b_sum, idx, s_sel,
                                                                ctx);
  return cudaGetLastError();
}

}  // namespace hils
