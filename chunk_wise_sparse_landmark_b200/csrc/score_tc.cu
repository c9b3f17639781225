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
// four heads' query tiles are written once into tensor memory (256 columns)
// and serve as the A operand of every MMA; k' tiles of 64 chunks x 128 for the
// four heads (64 KB) stream through a 2-stage TMA ring (128-byte swizzle,
// chunks past C read as zero) into one 4 x 64-column fp32 accumulator.  A
// thread that issues tcgen05.mma gets one instruction through every ~130
// cycles whatever its N, so each head has its own issuing warp (warps 0..3,
// lane 0; warp 0 also drives the TMA ring): together they keep the tensor
// pipe busy.  Warps 4..11 are the epilogue: two threads per position (its
// TMEM lane), one per 32-chunk half of each tile.
//
// Selection is exact and deterministic.  Pass 1 streams every tile; each
// epilogue thread keeps the multiset of the KT >= K largest group scores of
// its half, sorted in registers.  The candidates of a tile that beat the
// list's current KT-th value are appended to the thread's column of a
// shared-memory buffer; once some lane of the warp holds 32 of them, the warp
// sorts 32 buffered values per lane with a bitonic network and merges them
// into its list (a handful of merges per row instead of one insertion per
// candidate).  After the last tile the row's
// threshold tau (its K-th largest score) is the minimum over j < K of
// max(a_j, b_{K-1-j}) for the two halves' sorted lists a, b, and A = the
// number of scores above tau.  Pass 2 recomputes the same tiles (same
// instructions, bit-identical scores) and emits, in ascending chunk order,
// every candidate scoring above tau plus the first K - A scoring exactly tau
// (ties go to the smaller chunk), with each head's own s^.  Pass 2 reads the
// four heads' scores from TMEM once per tile and releases the accumulator
// before selecting, so that the next tile's MMAs overlap its selection and
// emission.  For K <= 32 the chosen chunks and scores are staged in shared
// memory and leave, after the last tile, as whole rows (consecutive threads,
// consecutive addresses).
#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int D = 128, G = 4;
constexpr int MQ = 128;   // positions per CTA (MMA M, TMEM lanes)
constexpr int TCH = 64;   // chunks per tile (MMA N)
constexpr int HALF = TCH / 2;
constexpr int NST = 2;    // k' ring stages (3 measured 0.5 ms slower with an earlier epilogue; beside
                          // the staging area of K <= 32 they no longer fit in shared memory)
constexpr int KMAX = 64;
constexpr int NMMA = G;   // MMA-issuing warps, one per head
constexpr int EPI = 256;  // epilogue threads
constexpr int THREADS = 32 * NMMA + EPI;
constexpr int CAP = 64;   // buffered candidates per epilogue thread (<= 31 carried + one tile's 32)
constexpr int RS = MQ + 1;  // row stride of the staged selection (conflict-free both ways)
constexpr uint32_t BBOX = TCH * 128;       // one [64 chunks x 64 d] bf16 box
constexpr uint32_t BSTAGE = G * 2 * BBOX;  // 64 KB
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACOL = 0;    // A: head h at ACOL + 64 h
constexpr uint32_t DCOL = 256;  // D: head h at DCOL + 64 h

// staging of the chosen chunks in pass 2: scores [G][KT][RS], then chunks [KT][RS]
template <int KT>
constexpr int kSelFloats = KT <= 32 ? (G + 1) * KT * RS : 0;
template <int KT>
constexpr int kAreaFloats = kSelFloats<KT> > CAP * EPI ? kSelFloats<KT> : CAP * EPI;

template <int KT>
struct __align__(1024) SmemS {
  unsigned char b[NST][G][2][BBOX];
  // pass 1: candidate buffer [CAP][EPI]; after it the [32][MQ] half-merge area;
  // pass 2 (K <= 32): the staged selection
  float area[kAreaFloats<KT>];
  alignas(16) float bt[2][G][TCH];  // b' of the tile, by tile parity, head-major
  alignas(16) float btj[2][TCH][G];  // the same, heads innermost
  uint8_t cnt[2][2][2][MQ];       // pass 2, by tile parity: [half][above / equal][row]
  float tau[MQ];
  int nab[2][MQ];
  int nselr[MQ];
  uint64_t bfull[NST], bempty[NST], dfull, dempty, afull, done;
  uint32_t tmem;
};

HILS_DI void epi_barrier() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// barrier of the two epilogue warps that hold the same rows (lane quadrant qd)
HILS_DI void row_pair_barrier(int qd) { asm volatile("bar.sync %0, 64;" ::"r"(2 + qd) : "memory"); }
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

// sort 32 values descending in registers (bitonic network, 240 compare-exchanges)
HILS_DI void sort32_desc(float (&a)[32]) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int l = i ^ j;
        if (l > i) {
          const float x = a[i], y = a[l];
          const bool desc = (i & k) == 0;
          a[i] = desc ? fmaxf(x, y) : fminf(x, y);
          a[l] = desc ? fminf(x, y) : fmaxf(x, y);
        }
      }
}

// top (the KT largest so far, descending) <- the KT largest of top and b (32
// values, descending): the elementwise max of top and b reversed is bitonic and
// holds those KT values; a bitonic merge sorts it descending
template <int KT>
HILS_DI void merge_top(float (&top)[KT], const float (&b)[32]) {
#pragma unroll
  for (int i = 0; i < KT; ++i) {
    const int bi = KT - 1 - i;
    top[i] = fmaxf(top[i], bi < 32 ? b[bi] : -INFINITY);
  }
#pragma unroll
  for (int j = KT >> 1; j > 0; j >>= 1)
#pragma unroll
    for (int i = 0; i < KT; ++i) {
      const int l = i ^ j;
      if (l > i) {
        const float x = top[i], y = top[l];
        top[i] = fmaxf(x, y);
        top[l] = fminf(x, y);
      }
    }
}

template <int KT>
__global__ void __launch_bounds__(THREADS, 1)
    score_topk_tc_kernel(Shape s, const __grid_constant__ CUtensorMap tmk, const __nv_bfloat16* __restrict__ q,
                         const float* __restrict__ b_sum, int32_t* __restrict__ idx, float* __restrict__ s_sel,
                         DevCtx ctx) {
  extern __shared__ unsigned char smem_raw[];
  SmemS<KT>& sm = *reinterpret_cast<SmemS<KT>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y, b = blockIdx.z;
  const int i0 = blockIdx.x * MQ;
  const int K = s.K;
  const int last = min(i0 + MQ, s.N) - 1;
  const int ncand_max = max(0, last / 64 - s.nw + 1);
  const int T = (ncand_max + TCH - 1) / TCH;  // tiles per pass
  const int NIT = 2 * T;

  if (tid == 0) {
    for (int x = 0; x < NST; ++x) {
      mbar_init(&sm.bfull[x], 1);
      mbar_init(&sm.bempty[x], NMMA);
    }
    mbar_init(&sm.dfull, NMMA);
    mbar_init(&sm.dempty, EPI / 32);
    mbar_init(&sm.afull, EPI / 32);
    mbar_init(&sm.done, NMMA);
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

  if (warp < NMMA) {
    // ------------------------------------- MMA issue (+ TMA ring, warp 0) ---
    const int h = warp;
    int nprod = 0;  // items put into the ring (warp 0)
    auto produce = [&](int it) {
      const int t = it % T, sb = it % NST;
      if (lane == 0 && ctx.inject != 1) {
        mbar_arrive_expect_tx(&sm.bfull[sb], BSTAGE);
        for (int hh = 0; hh < G; ++hh) {
          const int z = b * s.Hq + g * G + hh;
          tma_load_3d(sm.b[sb][hh][0], &tmk, 0, t * TCH, z, &sm.bfull[sb]);
          tma_load_3d(sm.b[sb][hh][1], &tmk, 64, t * TCH, z, &sm.bfull[sb]);
        }
      }
      nprod = it + 1;
    };
    if (warp == 0) {
      if (lane == 0 && NIT > 0) prefetch_tmap(&tmk);
      for (int it = 0; it < min(NST, NIT); ++it) produce(it);
      __syncwarp();
    }
    const uint32_t idesc = idesc_bf16_f32(MQ, TCH);
    bool ok = NIT == 0 || mbar_wait(&sm.afull, 0, ctx);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    for (int it = 0; it < NIT && ok; ++it) {
      const int sb = it % NST;
      ok = mbar_wait(&sm.bfull[sb], (it / NST) & 1, ctx);
      if (ok && it > 0) ok = mbar_wait(&sm.dempty, (it - 1) & 1, ctx);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t bdesc_addr = smem_u32(sm.b[sb][h][kk >> 2]) + (kk & 3) * 32;
          mma_ts(tmem + DCOL + h * 64, tmem + ACOL + h * 64 + kk * 8, sdesc_k_sw128(bdesc_addr), idesc,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(&sm.bempty[sb]);
        tc_commit(&sm.dfull);
      }
      __syncwarp();
      if (warp == 0 && it + NST < NIT) {
        // the stage is free once every head's MMAs of this tile have completed
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.bempty[sb], (it / NST) & 1, ctx));
        if (ok) produce(it + NST);
        __syncwarp();
      }
    }
    if (warp == 0 && lane == 0) {
      // copies still in flight land before the CTA may exit
      for (int x = 0; x < NST && x < nprod; ++x) mbar_wait(&sm.bfull[x], ((nprod - 1 - x) / NST) & 1, ctx);
    }
    // every MMA issued above has completed before the columns are released
    if (lane == 0) {
      tc_commit(&sm.done);
      mbar_wait(&sm.done, 0, ctx);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue ----
    const int e = warp - NMMA;        // 0..7
    const int hf = e >> 2;            // half of each tile: chunks [32 hf, 32 hf + 32)
    const int qd = warp & 3;          // TMEM lane quadrant of this warp
    const int r = qd * 32 + lane;     // row = TMEM lane
    const int et = e * 32 + lane;     // epilogue thread index
    const int i = i0 + r;
    const bool valid = i < s.N;
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    float(*mrg)[MQ] = reinterpret_cast<float(*)[MQ]>(&sm.area[0]);
    float* buf = &sm.area[et];  // this thread's candidate column: buf[x * EPI]
    float* sval = &sm.area[0];  // staged scores [G][KT][RS]
    int* sidx = reinterpret_cast<int*>(&sm.area[G * KT * RS]);  // staged chunks [KT][RS]
    constexpr bool kStaged = KT <= 32;
    // A: this row's scoring query, heads 2 hf and 2 hf + 1 -> TMEM
    for (int hh = 2 * hf; hh < 2 * hf + 2; ++hh) {
      const uint4* src =
          reinterpret_cast<const uint4*>(q + (((long long)b * s.Hq + g * G + hh) * s.N + (valid ? i : 0)) * D);
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
        tmem_st32(lane_addr + ACOL + hh * 64 + half * 32, w);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.afull);

    const int ncand = valid ? max(0, i / 64 - s.nw + 1) : 0;
    const float scale = s.scale;
    float top[KT];  // pass 1: this half's KT largest group scores, descending
#pragma unroll
    for (int j = 0; j < KT; ++j) top[j] = -INFINITY;
    float tau = -INFINITY;  // pass 2: the row's K-th largest group score
    int t_rem = 0;          // pass 2: scores equal to tau still to take
    int nsel = 0;
    int nb = 0;             // pass 1: candidates in this thread's buffer column
    const long long row_idx = (((long long)b * s.Hkv + g) * s.N + i) * K;
    bool ok = true;

    // b' of tile t for every head: thread et fetches head et / 64, chunk
    // et % 64, in two layouts (head-major for pass 1, heads innermost for
    // pass 2); the barrier of the landed vote publishes them.  The buffer of
    // this parity was last read two tiles ago, before the previous vote.
    auto load_bias = [&](int t) -> float {
      const int bh = et >> 6, bj = et & 63, bc = t * TCH + bj;
      return bc < s.C ? __ldg(b_sum + ((long long)b * s.Hq + g * G + bh) * s.C + bc) : 0.f;
    };
    auto stage_bias = [&](float bval, int par) {
      const int bh = et >> 6, bj = et & 63;
      sm.bt[par][bh][bj] = bval;
      sm.btj[par][bj][bh] = bval;
    };
    float bnext = T > 0 ? load_bias(0) : 0.f;  // b' of the next tile, fetched a tile ahead

    // pass 1
    for (int it = 0; it < T; ++it) {
      const int t = it, par = it & 1;
      const int c0 = t * TCH + hf * HALF;  // first chunk of this thread's half
      const float bval = bnext;
      bnext = load_bias(t + 1 < T ? t + 1 : 0);  // pass 2 starts again at tile 0
      stage_bias(bval, par);
      const bool landed = mbar_wait(&sm.dfull, it & 1, ctx);
      if (!epi_all(landed)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // group score of each chunk of this half: max over heads of v * scale + b'
      float gv[HALF];
      constexpr int HW = KT <= 32 ? 2 : 1;  // heads loaded per TMEM wait
#pragma unroll
      for (int h0 = 0; h0 < G; h0 += HW) {
        uint32_t v[HW][HALF];
#pragma unroll
        for (int u = 0; u < HW; ++u) tmem_ld32(lane_addr + DCOL + (h0 + u) * 64 + hf * HALF, v[u]);
        tmem_wait_ld();
        if (h0 + HW == G) {
          // the accumulator is read: the next tile's MMAs may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.dempty);
        }
#pragma unroll
        for (int u = 0; u < HW; ++u) {
          const int hh = h0 + u;
          const float4* bt4 = reinterpret_cast<const float4*>(&sm.bt[par][hh][hf * HALF]);
#pragma unroll
          for (int j4 = 0; j4 < HALF / 4; ++j4) {
            const float4 bb = bt4[j4];
            const float x0 = __fmaf_rn(__uint_as_float(v[u][4 * j4 + 0]), scale, bb.x);
            const float x1 = __fmaf_rn(__uint_as_float(v[u][4 * j4 + 1]), scale, bb.y);
            const float x2 = __fmaf_rn(__uint_as_float(v[u][4 * j4 + 2]), scale, bb.z);
            const float x3 = __fmaf_rn(__uint_as_float(v[u][4 * j4 + 3]), scale, bb.w);
            gv[4 * j4 + 0] = hh == 0 ? x0 : fmaxf(gv[4 * j4 + 0], x0);
            gv[4 * j4 + 1] = hh == 0 ? x1 : fmaxf(gv[4 * j4 + 1], x1);
            gv[4 * j4 + 2] = hh == 0 ? x2 : fmaxf(gv[4 * j4 + 2], x2);
            gv[4 * j4 + 3] = hh == 0 ? x3 : fmaxf(gv[4 * j4 + 3], x3);
          }
        }
      }
      // candidates above the list's current KT-th value join the buffer; a
      // warp merges when any lane has a tile's worth (32) buffered, and the
      // last tile flushes everything (at most two merges, nb <= 63)
      const float thr = top[KT - 1];
      const int jn = ncand - c0;
#pragma unroll
      for (int j = 0; j < HALF; ++j) {
        if (j < jn && gv[j] > thr) {
          buf[nb * EPI] = gv[j];
          ++nb;
        }
      }
      const bool flush = t == T - 1;  // CTA-uniform
      while (__any_sync(0xffffffffu, flush ? nb > 0 : nb >= HALF)) {
        float bb[HALF];
#pragma unroll
        for (int x = 0; x < HALF; ++x) bb[x] = x < nb ? buf[x * EPI] : -INFINITY;
        sort32_desc(bb);
        merge_top<KT>(top, bb);
        const int rest = max(nb - HALF, 0);
#pragma unroll
        for (int x = 0; x < HALF - 1; ++x)
          if (x < rest) buf[x * EPI] = buf[(HALF + x) * EPI];
        nb = rest;
      }
      if (t == T - 1) {
        // row threshold from the two halves' sorted lists a (half 0), b (half 1):
        // tau = min_{j<K} max(a_j, b_{K-1-j})
        epi_barrier();  // buffer reads done before the area is reused
        float tmin = INFINITY;
#pragma unroll
        for (int rd = 0; rd < (KT + 31) / 32; ++rd) {
          if (hf == 1) {
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if (32 * rd + x < KT) mrg[x][r] = top[min(32 * rd + x, KT - 1)];
          }
          epi_barrier();
          if (hf == 0) {
#pragma unroll
            for (int j = 0; j < KT; ++j) {
              const int jb = K - 1 - j - 32 * rd;
              if (j < K && jb >= 0 && jb < 32) tmin = fminf(tmin, fmaxf(top[j], mrg[jb][r]));
            }
          }
          epi_barrier();
        }
        if (hf == 0) sm.tau[r] = tmin;
        epi_barrier();
        tau = sm.tau[r];
        int above = 0;
#pragma unroll
        for (int j = 0; j < KT; ++j) above += top[j] > tau ? 1 : 0;
        sm.nab[hf][r] = above;
        epi_barrier();
        t_rem = max(0, K - (sm.nab[0][r] + sm.nab[1][r]));
      }
    }

    // pass 2: the four heads' scores are read from TMEM once per tile and the
    // accumulator is released at once, so that the next tile's MMAs overlap the
    // selection and the emission below
    for (int it = T; it < 2 * T && ok; ++it) {
      const int t = it - T, par = it & 1;
      const int c0 = t * TCH + hf * HALF;
      const float bval = bnext;
      if (t + 1 < T) bnext = load_bias(t + 1);
      stage_bias(bval, par);
      const bool landed = mbar_wait(&sm.dfull, it & 1, ctx);
      if (!epi_all(landed)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[G][HALF];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) tmem_ld32(lane_addr + DCOL + hh * 64 + hf * HALF, v[hh]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.dempty);
      // the same group scores as pass 1 (same operations, same order)
      const float4* bq = reinterpret_cast<const float4*>(&sm.btj[par][hf * HALF][0]);
      uint32_t gt = 0u, eq = 0u;
      const int jn = ncand - c0;  // candidates of this half: j < jn
#pragma unroll
      for (int j = 0; j < HALF; ++j) {
        const float4 bb = bq[j];
        float x = __fmaf_rn(__uint_as_float(v[0][j]), scale, bb.x);
        x = fmaxf(x, __fmaf_rn(__uint_as_float(v[1][j]), scale, bb.y));
        x = fmaxf(x, __fmaf_rn(__uint_as_float(v[2][j]), scale, bb.z));
        x = fmaxf(x, __fmaf_rn(__uint_as_float(v[3][j]), scale, bb.w));
        if (j < jn) {
          if (x > tau) gt |= 1u << j;
          else if (x == tau) eq |= 1u << j;
        }
      }
      // the two threads of a row (warps qd and qd + 4) exchange their counts
      sm.cnt[par][hf][0][r] = (uint8_t)__popc(gt);
      sm.cnt[par][hf][1][r] = (uint8_t)__popc(eq);
      row_pair_barrier(qd);
      const int g0 = sm.cnt[par][0][0][r], e0 = sm.cnt[par][0][1][r];
      const int g1 = sm.cnt[par][1][0][r], e1 = sm.cnt[par][1][1][r];
      const int take0 = min(e0, t_rem), take1 = min(e1, t_rem - take0);
      uint32_t sel = gt, em = eq;
      for (int x = 0; x < (hf ? take1 : take0); ++x) {
        sel |= em & (0u - em);
        em &= em - 1u;
      }
      const int base = nsel + (hf ? g0 + take0 : 0);
      nsel += g0 + take0 + g1 + take1;
      t_rem -= take0 + take1;
      if (__any_sync(0xffffffffu, sel != 0u)) {
        // the chosen chunks of this half take slots base, base + 1, ... in
        // ascending chunk order; one predicated step per chunk, from registers
        // (measured at 128K: a select tree per chosen chunk and head, fed by a
        // second TMEM read, was 2.4 ms of the kernel)
        int slot = base;
#pragma unroll
        for (int j = 0; j < HALF; ++j) {
          if (sel & (1u << j)) {
            if (slot < K) {
              // b' from the head-major copy: the four loads of the mask loop
              // above are not kept alive across it
              const float* bh = &sm.bt[par][0][hf * HALF + j];
              const float y[G] = {__fmaf_rn(__uint_as_float(v[0][j]), scale, bh[0]),
                                  __fmaf_rn(__uint_as_float(v[1][j]), scale, bh[TCH]),
                                  __fmaf_rn(__uint_as_float(v[2][j]), scale, bh[2 * TCH]),
                                  __fmaf_rn(__uint_as_float(v[3][j]), scale, bh[3 * TCH])};
              if constexpr (kStaged) {
                sidx[slot * RS + r] = c0 + j;
#pragma unroll
                for (int hh = 0; hh < G; ++hh) sval[(hh * KT + slot) * RS + r] = y[hh];
              } else {
                idx[row_idx + slot] = c0 + j;
#pragma unroll
                for (int hh = 0; hh < G; ++hh) s_sel[(((long long)b * s.Hq + g * G + hh) * s.N + i) * K + slot] = y[hh];
              }
            }
            ++slot;
          }
        }
      }
    }
    if (valid && ok && hf == 0 && nsel != min(ncand, K)) raise_status(ctx, kStatusBadIndex);
    if constexpr (kStaged) {
      // the staged rows leave whole: element f = row * K + slot of the CTA's
      // rows, consecutive threads at consecutive addresses; slots past the
      // row's selection get -1 / -inf
      if (hf == 0) sm.nselr[r] = min(nsel, K);
      epi_barrier();
      if (ok) {
        const int tot = (min(i0 + MQ, s.N) - i0) * K;
        int32_t* idx0 = idx + (((long long)b * s.Hkv + g) * s.N + i0) * K;
        for (int f = et; f < tot; f += EPI) {
          const int rr = f / K, k = f - rr * K;
          const bool on = k < sm.nselr[rr];
          idx0[f] = on ? sidx[k * RS + rr] : -1;
#pragma unroll
          for (int hh = 0; hh < G; ++hh)
            s_sel[(((long long)b * s.Hq + g * G + hh) * s.N + i0) * K + f] =
                on ? sval[(hh * KT + k) * RS + rr] : -INFINITY;
        }
      }
    } else if (valid && ok && hf == 0) {
      nsel = min(nsel, K);
      for (int x = nsel; x < K; ++x) {
        idx[row_idx + x] = -1;
#pragma unroll
        for (int hh = 0; hh < G; ++hh) s_sel[(((long long)b * s.Hq + g * G + hh) * s.N + i) * K + x] = -INFINITY;
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

template <int KT>
constexpr size_t kSmemBytes = sizeof(SmemS<KT>) + 1024;
static_assert(kSmemBytes<16> <= 232448 && kSmemBytes<32> <= 232448 && kSmemBytes<64> <= 232448,
              "score kernel shared memory above the 227 KB a CTA may use");

template <int KT>
cudaError_t launch_kt(const Shape& s, const CUtensorMap& tmk, const void* q, const float* b_sum, int32_t* idx,
                      float* s_sel, cudaStream_t st, const DevCtx& ctx) {
  cudaError_t e = ensure_dynamic_smem((const void*)score_topk_tc_kernel<KT>, (int)kSmemBytes<KT>);
  if (e != cudaSuccess) return e;
  dim3 grid((s.N + MQ - 1) / MQ, s.Hkv, s.B);
  score_topk_tc_kernel<KT><<<grid, THREADS, kSmemBytes<KT>, st>>>(s, tmk, (const __nv_bfloat16*)q, b_sum, idx, s_sel,
                                                               ctx);
  return cudaGetLastError();
}

}  // namespace

size_t score_tc_workspace(const Shape&) { return 0; }

cudaError_t launch_score_topk_tc(const Shape& s, const void* q, const void* k_sum, const float* b_sum, int32_t* idx,
                                 float* s_sel, cudaStream_t st, const DevCtx& ctx) {
  if (s.d != D || s.G != G || s.K > KMAX || s.K < 1 || s.S != 64) return cudaErrorNotSupported;
  CUtensorMap tmk;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)(s.C > 0 ? s.C : 1), (uint64_t)s.B * s.Hq};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)(s.C > 0 ? s.C : 1) * D * 2};
  const uint32_t box[3] = {64, TCH, 1};
  cudaError_t e = make_tmap_bf16(&tmk, k_sum, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  if (s.K <= 16) return launch_kt<16>(s, tmk, q, b_sum, idx, s_sel, st, ctx);
  if (s.K <= 32) return launch_kt<32>(s, tmk, q, b_sum, idx, s_sel, st, ctx);
  return launch_kt<64>(s, tmk, q, b_sum, idx, s_sel, st, ctx);
}

}  // namespace hils
