// Selected-chunk attention, chunk-major, on the tcgen05 tensor cores (bf16
// prefill, d = 128, S = 64, G = 4).
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method): every selected chunk c of position i is attended on its own,
//   O_{i,c} = sum_{j in c} softmax_{j in c}(q_i.k_j * scale) v_j,
// and the chunk outputs are fused with weights exp(s^_{i,c}) / Z^_i.  O_{i,c}
// depends on nothing but q_i and chunk c, so the pairs (i, c) can be computed
// in any grouping.  This file groups them by chunk: the positions that chose
// chunk c (of one KV group) are gathered 32 at a time (x 4 heads = 128 query
// rows, the MMA's M), and chunk c's K and V tiles are loaded once for all of
// them:
//
//   S (128 rows x 64 keys)  = Q_rows (128 x d) . K_c^T        tcgen05, fp32 in TMEM
//   P = softmax over the 64 keys of each row, bf16, written back into TMEM
//   O (128 rows x 128 d)    = P (128 x 64) . V_c (64 x d)     tcgen05, fp32 in TMEM
//
// O is stored as one 1 KB bf16 record per (position, slot k of its selection
// list; heads innermost) -- the "partial" -- and attn_window.cu attends the
// window with its exact softmax terms and fuses the partials with the exp(s^)
// weights.
//
// Why chunk-major: on the pages' i.i.d.-like workloads adjacent positions
// share almost none of their selected chunks, so a position-major kernel
// moves a 32 KB K/V tile per (position pair, chunk) into shared memory and
// reads it back for 8 query rows.  Grouped by chunk, a tile serves ~100+ rows
// and the work becomes dense tensor-core tiles; the price is the gathered
// query rows (1 KB per pair, mostly L2 hits) and the partial records (1 KB per
// pair written here, read once by the fusion kernel).
//
// Bucketing (three small kernels per position tile): count the pairs
// per (sequence, KV group, chunk) bucket, scan the counts into bucket offsets
// and item offsets (one item = up to 32 positions of one bucket), scatter the
// pairs into their buckets and write the item table.  The order of the pairs
// inside a bucket depends on atomic arrival order, but no result does: every
// output row is computed by the same instructions wherever it sits in a tile.
//
// CTA layout (one persistent CTA per SM, 576 threads, items dealt round-robin):
//   warp 0      TMA loads of the chunk's K and V tiles (128-byte swizzle); 6 stages
//   warp 1      tcgen05.mma issue (one thread); S and O double-buffered in TMEM
//   warps 2-9   query rows: two groups of four warps take alternate items;
//               each thread owns one row (its TMEM lane), loads its 256 bytes
//               from the tile's regrouped copy (regroup_q_kernel: a
//               position's 4 heads side by side) with 32-byte loads and
//               stores them into TMEM, where
//               they are the A operand of S = Q K^T (no shared-memory staging
//               and no swizzle for the gathered rows)
//   warps 10-13 softmax: TMEM S row -> max, exp2 -> normalised bf16 P row,
//               written back into the first half of the row's S columns; the
//               second MMA reads P from TMEM (no shared-memory traffic)
//   warps 14-17 epilogue: TMEM O row -> bf16 partial record (a position's
//               4 head rows are adjacent lanes: 128-byte lines per store)
// 18 warps: the register file is split across the four sub-partitions, so
// 96 registers per thread is the most that fits.
//
// Measured on B200 at 128K:
//   - Staging the gathered rows in shared memory with 16-byte cp.async held
//     only ~20 KB in flight per SM and set a period of ~5K cycles per item;
//     32-byte loads into registers keep far more in flight.
//   - A build that skipped the record stores ran 13 ms faster (36.1 -> 23.2 ms
//     for the attention call) while the records were written as 16-byte halves
//     of sectors from separate passes.  Writing each 64-column half of a row as
//     one contiguous 128-byte run took the attention to 30.9 ms.
//   - Records with heads innermost (8 whole lines per warp store) and
//     regrouped query rows (8 lines per warp load instead of 32) took the
//     chunk kernel from ~15.6 to 9.5 ms.
//   - A second MMA-issuing thread, a second softmax group and a second
//     epilogue group each changed nothing measurable.
//   - Copy-engine gathers issued from all lanes of a warp (one tile::gather4 or
//     one 256-byte bulk copy per row) did not complete, and are not used.
// Every wait is bounded (status word + early return), see common.cuh.
#include <algorithm>
#include <mutex>

#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int D = 128, S = 64, G = 4;
constexpr int PPI = 32;          // positions per item
constexpr int MR = PPI * G;      // query rows per item (MMA M)
constexpr int NQS = 2;           // query-row stages (TMEM), one per row group
constexpr int NKV = 6;           // K/V stages
constexpr int NST = 2;           // S / P / O stages
constexpr uint32_t BOX = S * 128;     // [64 keys x 64 d] bf16 (8 KB)
constexpr int THREADS = 18 * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t OCOL = 0;     // O of stage st at OCOL + 128 st
constexpr uint32_t SCOL = 256;   // S of stage st at SCOL + 64 st
constexpr uint32_t QCOL = 384;   // query rows of stage sq at QCOL + 64 sq (bf16 pairs)
constexpr int KMAX = 64;

struct __align__(1024) SmemC {
  unsigned char k[NKV][2][BOX];     // [d half][key][128 B]
  unsigned char v[NKV][2][BOX];     // [d half][key][128 B]
  uint64_t qfull[NQS], qempty[NQS], kvfull[NKV], kvempty[NKV];
  uint64_t sfull[NST], sfree[NST], pfull[NST], ofull[NST], ofree[NST], done;
  uint32_t tmem;
};
constexpr size_t kSmemBytes = sizeof(SmemC) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

HILS_DI void ldg32(const void* p, uint32_t (&w)[8]) {
  asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
               : "l"(p));
}
// 32-byte global store (address 32-byte aligned)
HILS_DI void stg32(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}
struct Item {
  int bg, c, s0, n;
};

__global__ void __launch_bounds__(THREADS, 1)
    attn_chunk_kernel(Shape s, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                      const int* __restrict__ ioff, const int4* __restrict__ items, const int* __restrict__ ent,
                      int PT, const __nv_bfloat16* __restrict__ qg, __nv_bfloat16* __restrict__ part, DevCtx ctx) {
  extern __shared__ unsigned char smem_raw[];
  SmemC& sm = *reinterpret_cast<SmemC*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int U = s.B * s.Hkv * s.C;
  const int nitems = __ldg(ioff + U);
  const int bid = blockIdx.x, nb = gridDim.x;
  const int nmine = nitems > bid ? (nitems - 1 - bid) / nb + 1 : 0;
  // item record: bucket u = bg * C + c, first pair s0, pair count n (<= 32)
  auto item_of = [&](int it) -> Item {
    Item r{0, 0, 0, 0};
    if (it < nmine) {
      const int4 e = __ldg(items + bid + it * nb);
      r.bg = e.x / s.C;
      r.c = e.x - r.bg * s.C;
      r.s0 = e.y;
      r.n = e.z;
    }
    return r;
  };

  if (tid == 0) {
    for (int x = 0; x < NQS; ++x) {
      mbar_init(&sm.qfull[x], 4);
      mbar_init(&sm.qempty[x], 1);
    }
    for (int x = 0; x < NKV; ++x) {
      mbar_init(&sm.kvfull[x], 1);
      mbar_init(&sm.kvempty[x], 1);
    }
    for (int x = 0; x < NST; ++x) {
      mbar_init(&sm.sfull[x], 1);
      mbar_init(&sm.sfree[x], 1);
      mbar_init(&sm.pfull[x], 4);
      mbar_init(&sm.ofull[x], 1);
      mbar_init(&sm.ofree[x], 4);
    }
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
    // --------------------------------------------------------- K/V loads ----
    if (lane == 0) {
      bool ok = true;
      int it = 0;
      if (nmine > 0) {
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
      }
      Item nx = item_of(0);
      for (; it < nmine; ++it) {
        const int sk = it % NKV;
        const Item im = nx;
        nx = item_of(it + 1);
        if (it >= NKV) ok = mbar_wait(&sm.kvempty[sk], ((it / NKV) - 1) & 1, ctx);
        if (!ok) break;
        if (ctx.inject != 1) {
          mbar_arrive_expect_tx(&sm.kvfull[sk], 4 * BOX);
          tma_load_3d(sm.k[sk][0], &tmk, 0, im.c * S, im.bg, &sm.kvfull[sk]);
          tma_load_3d(sm.k[sk][1], &tmk, 64, im.c * S, im.bg, &sm.kvfull[sk]);
          tma_load_3d(sm.v[sk][0], &tmv, 0, im.c * S, im.bg, &sm.kvfull[sk]);
          tma_load_3d(sm.v[sk][1], &tmv, 64, im.c * S, im.bg, &sm.kvfull[sk]);
        }
      }
      // the copies issued last land before the CTA exits, whichever role gave
      // up first (their phases completed long ago on the normal path)
      if (ctx.inject != 1)
        for (int j = max(0, it - NKV); j < it; ++j) mbar_wait(&sm.kvfull[j % NKV], (j / NKV) & 1, ctx);
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issue ----
    if (lane == 0) {
      const uint32_t id1 = idesc_bf16_f32(MR, S);
      const uint32_t id2 = idesc_bf16_f32(MR, D) | (1u << 16);  // B (V) is MN-major
      auto mma1 = [&](int j) -> bool {
        const int st = j % NST, sq = j % NQS, sk = j % NKV;
        if (!mbar_wait(&sm.qfull[sq], (j / NQS) & 1, ctx)) return false;
        if (!mbar_wait(&sm.kvfull[sk], (j / NKV) & 1, ctx)) return false;
        if (j >= NST && !mbar_wait(&sm.sfree[st], ((j / NST) - 1) & 1, ctx)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = sdesc_k_sw128(smem_u32(sm.k[sk][kk >> 2]) + (kk & 3) * 32);
          mma_ts(tmem + SCOL + 64 * st, tmem + QCOL + 64 * sq + 8 * kk, bd, id1, kk > 0 ? 1u : 0u);
        }
        tc_commit(&sm.sfull[st]);
        tc_commit(&sm.qempty[sq]);
        return true;
      };
      auto mma2 = [&](int j) -> bool {
        const int st = j % NST, sk = j % NKV;
        if (!mbar_wait(&sm.pfull[st], (j / NST) & 1, ctx)) return false;
        if (j >= NST && !mbar_wait(&sm.ofree[st], ((j / NST) - 1) & 1, ctx)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = sdesc_mn_sw128(smem_u32(sm.v[sk][0]) + kk * 2048, BOX, 1024);
          mma_ts(tmem + OCOL + 128 * st, tmem + SCOL + 64 * st + 8 * kk, bd, id2, kk > 0 ? 1u : 0u);
        }
        tc_commit(&sm.ofull[st]);
        tc_commit(&sm.kvempty[sk]);
        tc_commit(&sm.sfree[st]);  // P (in the S columns) has been read
        return true;
      };
      // S of item j + 1 is computed while the softmax of item j runs
      bool ok = nmine == 0 || mma1(0);
      for (int it = 0; it < nmine && ok; ++it) {
        if (it + 1 < nmine) ok = mma1(it + 1);
        if (ok) ok = mma2(it);
      }
      // every MMA issued above has completed before the columns are released
      tc_commit(&sm.done);
      mbar_wait(&sm.done, 0, ctx);
    }
    __syncwarp();
  } else if (warp < 10) {
    // -------------------------------------------------------- query rows ----
    // Group wg (warps 2-5 or 6-9) takes items wg, wg + 2, ...; thread = TMEM
    // lane = row r = 4 j + h: head h of the item's position j (rows past the
    // item's count are zero).  The rows come from the tile's regrouped copy,
    // where a position's 4 heads sit side by side in 32-byte pieces, so each
    // warp load reads 8 whole 128-byte lines (from q itself, 4 head planes
    // apart, it touched 32).  The 256-byte row is loaded before the stage is
    // known to be free, so the loads of one item overlap the wait for it.
    // Item metadata: records two items ahead, entries one item ahead.
    const int wg = (warp - 2) >> 2, qw = warp & 3, row = 32 * qw + lane, jr = row >> 2, h = row & 3;
    const uint32_t lrow = (uint32_t)(32 * qw) << 16;
    Item m0 = item_of(wg), m1 = item_of(wg + 2);
    int e0 = jr < m0.n ? __ldg(ent + m0.s0 + jr) : 0;
    for (int it = wg; it < nmine; it += 2) {
      const int sq = it % NQS, li = it / NQS;
      const bool valid = jr < m0.n;
      // regrouped rows (regroup_q_kernel): piece x of head h at (4 x + h) * 16
      const __nv_bfloat16* src = qg + ((long long)m0.bg * PT + (e0 >> 6)) * (G * D) + h * 16;
      uint32_t w[64];
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        uint32_t t8[8];
        if (valid) {
          ldg32(src + 64 * x, t8);
        } else {
#pragma unroll
          for (int y = 0; y < 8; ++y) t8[y] = 0u;
        }
#pragma unroll
        for (int y = 0; y < 8; ++y) w[8 * x + y] = t8[y];
      }
      e0 = jr < m1.n ? __ldg(ent + m1.s0 + jr) : 0;
      m0 = m1;
      m1 = item_of(it + 4);
      const bool ok = li == 0 || mbar_wait(&sm.qempty[sq], (li - 1) & 1, ctx);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t* w0 = w;
      tmem_st32(tmem + lrow + QCOL + 64 * sq, *reinterpret_cast<uint32_t(*)[32]>(w0));
      tmem_st32(tmem + lrow + QCOL + 64 * sq + 32, *reinterpret_cast<uint32_t(*)[32]>(w0 + 32));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.qfull[sq]);
    }
  } else if (warp < 14) {
    // ----------------------------------------------------------- softmax ----
    const int qw = warp & 3, row = 32 * qw + lane;
    const uint32_t lrow = (uint32_t)(32 * qw) << 16;
    const float sl2 = s.scale * kLog2e;
    bool ok = true;
    for (int it = 0; it < nmine; ++it) {
      const int st = it % NST;
      ok = mbar_wait(&sm.sfull[st], (it / NST) & 1, ctx);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tmem + lrow + SCOL + 64 * st, r0);
      tmem_ld32(tmem + lrow + SCOL + 64 * st + 32, r1);
      tmem_wait_ld();
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) mx = fmaxf(mx, fmaxf(__uint_as_float(r0[j]), __uint_as_float(r1[j])));
      const float base = mx * sl2;
      float l = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float e0 = exp2f(fmaf(__uint_as_float(r0[j]), sl2, -base));
        const float e1 = exp2f(fmaf(__uint_as_float(r1[j]), sl2, -base));
        r0[j] = __float_as_uint(e0);
        r1[j] = __float_as_uint(e1);
        l += e0 + e1;
      }
      const float inv = 1.f / l;
      // P row: keys 2c, 2c + 1 in column c (bf16 pairs), over S's first 32
      // columns; keys 0-31 (r0) and 32-63 (r1) in two 16-column stores
      uint32_t pw[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) pw[c] = pack_bf16x2(__uint_as_float(r0[2 * c]) * inv, __uint_as_float(r0[2 * c + 1]) * inv);
      tmem_st16(tmem + lrow + SCOL + 64 * st, pw);
#pragma unroll
      for (int c = 0; c < 16; ++c) pw[c] = pack_bf16x2(__uint_as_float(r1[2 * c]) * inv, __uint_as_float(r1[2 * c + 1]) * inv);
      tmem_st16(tmem + lrow + SCOL + 64 * st + 16, pw);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.pfull[st]);
    }
  } else {
    // ---------------------------------------------------------- epilogue ----
    // Partial record of (position, slot k): 1 KB of bf16, [unit u][head][32 B]
    // with u = 4 h2 + r / 2 (8 units of 128 bytes, heads innermost).  Unit
    // u's 32 bytes of a head hold pieces r and r + 1 of the head's 64-column
    // half h2 (r even); in piece r, element 4 a + t holds d = 64 h2 + 32 a +
    // r + 8 t (a = 0..1, t = 0..3): the values d = r (mod 8) of one half, the
    // unit of one fusion-kernel lane.  The 4 head rows of a position are 4
    // adjacent lanes, so each warp store writes 8 whole 128-byte lines.
    // Measured at 128K: head-major records (each warp store touching 32
    // lines) cost ~7 ms of the attention; item-major blocks of 128 rows (one
    // 512-byte run per store) were as fast to write but left the record reader
    // with 64-byte pieces 2 KB apart (17.5 ms against 13 ms); staging in
    // shared memory for 512-byte runs (41 ms, with spills) and bulk copies of
    // 1 KB records (32 ms) were slower.  Item metadata is fetched ahead.
    const int qw = warp & 3, row = 32 * qw + lane, jr = row >> 2, h = row & 3;
    const uint32_t lrow = (uint32_t)(32 * qw) << 16;
    Item m0 = item_of(0), m1 = item_of(1);
    int e0 = jr < m0.n ? __ldg(ent + m0.s0 + jr) : 0;
    for (int it = 0; it < nmine; ++it) {
      const int st = it % NST;
      const Item im = m0;
      const int e = e0;
      e0 = jr < m1.n ? __ldg(ent + m1.s0 + jr) : 0;
      m0 = m1;
      m1 = item_of(it + 2);
      const bool valid = jr < im.n;
      __nv_bfloat16* dst = part + (((long long)im.bg * PT + (e >> 6)) * s.K + (e & 63)) * (G * D) + h * 16;
      const bool ok = mbar_wait(&sm.ofull[st], (it / NST) & 1, ctx);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem + lrow + OCOL + 128 * st + 64 * pr, v0);
        tmem_ld32(tmem + lrow + OCOL + 128 * st + 64 * pr + 32, v1);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int r = 0; r < 8; r += 2) {
            uint32_t o[8];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              o[4 * u + 0] = pack_bf16x2(__uint_as_float(v0[r + u]), __uint_as_float(v0[r + u + 8]));
              o[4 * u + 1] = pack_bf16x2(__uint_as_float(v0[r + u + 16]), __uint_as_float(v0[r + u + 24]));
              o[4 * u + 2] = pack_bf16x2(__uint_as_float(v1[r + u]), __uint_as_float(v1[r + u + 8]));
              o[4 * u + 3] = pack_bf16x2(__uint_as_float(v1[r + u + 16]), __uint_as_float(v1[r + u + 24]));
            }
            stg32(dst + (4 * pr + r / 2) * (G * 16), o);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.ofree[st]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// The query rows of positions [t0, t0 + np), regrouped per KV group as
// qg[bg][p - t0][x][h][16 elements] (bg stride PT positions): 32-byte piece x
// of the G = 4 heads side by side (1 KB per position).  One warp per (bg, position): lane 4 x + h
// reads piece x of head h and the warp writes the position's 1 KB at once.
__global__ void __launch_bounds__(256) regroup_q_kernel(Shape s, const __nv_bfloat16* __restrict__ q, int t0, int np,
                                                        int PT, __nv_bfloat16* __restrict__ qg) {
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= (long long)s.B * s.Hkv * np) return;
  const int bg = (int)(w / np), pl = (int)(w - (long long)bg * np);
  const int b = bg / s.Hkv, g = bg - b * s.Hkv, x = lane >> 2, h = lane & 3;
  uint32_t t8[8];
  ldg32(q + ((long long)(b * s.Hq + g * G + h) * s.N + t0 + pl) * D + 16 * x, t8);
  stg32(qg + ((long long)bg * PT + pl) * (G * D) + lane * 16, t8);
}

// ------------------------------------------------------------ bucketing ----
// The lists of a position tile [t0, t0 + np): list r = bg * np + pl holds the
// K entries of position t0 + pl in KV group bg.  One warp reads one list
// (lane j: entries j and j + 32) and keeps the entries that have the list
// form (accept_list_warp, common.cuh); the fusion kernel applies the same rule
// before it fuses the records, so both agree on every pair.
HILS_DI void list_of(const Shape& s, const int32_t* __restrict__ idx, int t0, int np, long long r, int& bg, int& pl,
                     int& a, int& b, const DevCtx* report) {
  const int lane = threadIdx.x & 31;
  pl = (int)(r % np);
  bg = (int)(r / np);
  const int p = t0 + pl;
  const int32_t* L = idx + ((long long)bg * s.N + p) * s.K;
  a = lane < s.K ? __ldg(L + lane) : -1;
  b = lane + 32 < s.K ? __ldg(L + lane + 32) : -1;
  bool bad;
  accept_list_warp(a, b, s.K, max(0, p / S - s.nw + 1), bad);
  if (report && bad && lane == 0) raise_status(*report, kStatusBadIndex);
}

// Both passes run one block per (KV group bg, block of PB positions) and count
// into a shared histogram over the C chunks first, so that global atomics are
// one per (block, non-empty bucket) instead of one per pair (measured: ~0.25 ms
// per 32K-position tile with a global atomic per pair).
constexpr int PB = 1024;  // positions per bucketing block

HILS_DI void count_block(const Shape& s, const int32_t* __restrict__ idx, int t0, int np, int* hist,
                         const DevCtx* report) {
  const int bg = blockIdx.x / ((np + PB - 1) / PB), pb = blockIdx.x % ((np + PB - 1) / PB);
  const int p_end = min(np, (pb + 1) * PB), wpb = blockDim.x >> 5;
  for (int c = threadIdx.x; c < s.C; c += blockDim.x) hist[c] = 0;
  __syncthreads();
  for (int pl = pb * PB + (threadIdx.x >> 5); pl < p_end; pl += wpb) {
    int bgx, plx, a, b;
    list_of(s, idx, t0, np, (long long)bg * np + pl, bgx, plx, a, b, report);
    if (a >= 0) atomicAdd(hist + a, 1);
    if (b >= 0) atomicAdd(hist + b, 1);
  }
  __syncthreads();
}

__global__ void bucket_count_kernel(Shape s, const int32_t* __restrict__ idx, int t0, int np, int* __restrict__ cnt,
                                    DevCtx ctx) {
  extern __shared__ int hist[];
  count_block(s, idx, t0, np, hist, &ctx);
  const int bg = blockIdx.x / ((np + PB - 1) / PB);
  for (int c = threadIdx.x; c < s.C; c += blockDim.x)
    if (hist[c]) atomicAdd(cnt + bg * s.C + c, hist[c]);
}

// One block: exclusive scans of the bucket counts (pair offsets) and of their
// item counts ceil(n / 32) (item offsets); cnt becomes the scatter cursor.
__global__ void __launch_bounds__(1024) bucket_scan_kernel(int U, int* __restrict__ cnt, int* __restrict__ off,
                                                           int* __restrict__ ioff) {
  __shared__ int wa[32], wb[32];
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int per = (U + 1023) / 1024;
  const int u0 = min(U, t * per), u1 = min(U, u0 + per);
  int sa = 0, sb = 0;
  for (int u = u0; u < u1; ++u) {
    const int n = cnt[u];
    sa += n;
    sb += (n + PPI - 1) / PPI;
  }
  int ia = sa, ib = sb;  // inclusive warp scans
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int xa = __shfl_up_sync(0xffffffffu, ia, o), xb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia += xa;
      ib += xb;
    }
  }
  if (lane == 31) {
    wa[w] = ia;
    wb[w] = ib;
  }
  __syncthreads();
  if (w == 0) {
    int xa = wa[lane], xb = wb[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, xa, o), yb = __shfl_up_sync(0xffffffffu, xb, o);
      if (lane >= o) {
        xa += ya;
        xb += yb;
      }
    }
    wa[lane] = xa;  // inclusive over warps
    wb[lane] = xb;
  }
  __syncthreads();
  int ea = ia - sa + (w > 0 ? wa[w - 1] : 0), eb = ib - sb + (w > 0 ? wb[w - 1] : 0);
  for (int u = u0; u < u1; ++u) {
    const int n = cnt[u];
    off[u] = ea;
    ioff[u] = eb;
    cnt[u] = ea;
    ea += n;
    eb += (n + PPI - 1) / PPI;
  }
  if (t == 1023) {
    off[U] = ea;
    ioff[U] = eb;
  }
}

__global__ void bucket_scatter_kernel(Shape s, const int32_t* __restrict__ idx, int t0, int np,
                                      const int* __restrict__ off, const int* __restrict__ ioff, int* __restrict__ cur,
                                      int* __restrict__ ent, int4* __restrict__ items) {
  extern __shared__ int hist[];
  count_block(s, idx, t0, np, hist, nullptr);  // the count pass reported bad entries
  const int bg = blockIdx.x / ((np + PB - 1) / PB), pb = blockIdx.x % ((np + PB - 1) / PB);
  const int p_end = min(np, (pb + 1) * PB), wpb = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  // this block's range of every bucket: one global atomic per non-empty bucket
  for (int c = threadIdx.x; c < s.C; c += blockDim.x)
    if (hist[c]) hist[c] = atomicAdd(cur + bg * s.C + c, hist[c]);
  __syncthreads();
  for (int pl = pb * PB + (threadIdx.x >> 5); pl < p_end; pl += wpb) {
    int bgx, plx, a, b;
    list_of(s, idx, t0, np, (long long)bg * np + pl, bgx, plx, a, b, nullptr);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = h ? b : a;
      if (c < 0) continue;
      const int u = bg * s.C + c;
      const int slot = atomicAdd(hist + c, 1);  // shared cursor
      ent[slot] = (pl << 6) | (lane + 32 * h);
      const int rel = slot - __ldg(off + u);
      if (rel % PPI == 0)
        items[__ldg(ioff + u) + rel / PPI] = make_int4(u, slot, min(PPI, __ldg(off + u + 1) - slot), 0);
    }
  }
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// A side stream and its events per device, made on first use.  g_side_mu is
// held for a whole call's enqueue, so concurrent calls never record an event
// that another call is about to wait on.
struct Side {
  cudaStream_t st = nullptr;
  cudaEvent_t start = nullptr, next = nullptr, win = nullptr;
};
Side g_side[64];
std::mutex g_side_mu;

cudaError_t side_init(Side& sd) {
  cudaError_t e = cudaSuccess;
  if (!sd.st) e = cudaStreamCreateWithFlags(&sd.st, cudaStreamNonBlocking);
  if (e == cudaSuccess && !sd.start) e = cudaEventCreateWithFlags(&sd.start, cudaEventDisableTiming);
  if (e == cudaSuccess && !sd.next) e = cudaEventCreateWithFlags(&sd.next, cudaEventDisableTiming);
  if (e == cudaSuccess && !sd.win) e = cudaEventCreateWithFlags(&sd.win, cudaEventDisableTiming);
  return e;
}

// workspace pieces, in order
struct ChunkWs {
  size_t cnt, off, ioff, ent, items, qg, wst, part, total;
  int PT;
};

// Positions per tile: the fewest tiles whose partial records fit about
// kPartBudget bytes each, of equal size rounded up to a multiple of a chunk
// (the window pass's 32-position blocks then never straddle a tile).
constexpr size_t kPartBudget = size_t(8) << 30;
constexpr int kTileAlign = 64;

ChunkWs chunk_ws(const Shape& s) {
  ChunkWs w{};
  const size_t per_pos = (size_t)s.B * s.Hkv * s.K * G * D * 2;
  const long long cap = std::max<long long>(1, (long long)(kPartBudget / per_pos));
  const long long ntiles = (s.N + cap - 1) / cap;
  const long long pt = (s.N + ntiles - 1) / ntiles;
  w.PT = (int)((pt + kTileAlign - 1) / kTileAlign * kTileAlign);
  const size_t U = (size_t)s.B * s.Hkv * s.C;
  const size_t pairs = (size_t)s.B * s.Hkv * w.PT * s.K;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o += up256(bytes);
    return r;
  };
  w.cnt = take((U + 1) * 4);
  w.off = take((U + 1) * 4);
  w.ioff = take((U + 1) * 4);
  w.ent = take(pairs * 4);
  w.items = take((pairs / PPI + U + 1) * 16);
  w.qg = take((size_t)s.B * s.Hkv * w.PT * G * D * 2);
  w.wst = take(2 * window_state_bytes(s, w.PT));  // two tiles' window states
  w.part = take(pairs * G * D * 2);
  w.total = o;
  return w;
}

}  // namespace

size_t attn_prefill_tc_workspace(const Shape& s) {
  if (s.d != D || s.S != S || s.G != G || s.K > KMAX) return 0;
  return chunk_ws(s).total;
}

cudaError_t launch_attn_prefill_chunked(const Shape& s, const void* q, const void* k, const void* v,
                                        const int32_t* idx, const float* s_sel, void* out, void* ws,
                                        cudaStream_t st, const DevCtx& ctx) {
  if (s.d != D || s.S != S || s.G != G || s.K > KMAX) return cudaErrorNotSupported;
  const ChunkWs w = chunk_ws(s);
  unsigned char* W = (unsigned char*)ws;
  int* cnt = (int*)(W + w.cnt);
  int* off = (int*)(W + w.off);
  int* ioff = (int*)(W + w.ioff);
  int* ent = (int*)(W + w.ent);
  int4* items = (int4*)(W + w.items);
  __nv_bfloat16* qg = (__nv_bfloat16*)(W + w.qg);
  __nv_bfloat16* part = (__nv_bfloat16*)(W + w.part);
  const int U = s.B * s.Hkv * s.C;

  CUtensorMap tmk, tmv;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)s.N, (uint64_t)s.B * s.Hkv};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)s.N * D * 2};
  const uint32_t box[3] = {64, (uint32_t)S, 1};
  cudaError_t e = make_tmap_bf16(&tmk, k, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tmv, v, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = ensure_dynamic_smem((const void*)attn_chunk_kernel, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();

  // The window kernel of tile t + 1 runs on a side stream beside the fusion of
  // tile t (an HBM-bound kernel with room beside it on every SM); the chunk
  // kernel, which fills the SMs, runs alone.  Order per tile on `st`:
  // bucketing, regroup, [wait window(t)] chunk(t), [window(t + 1) starts on the
  // side stream], fusion(t).  The window state is double-buffered by tile.
  WindowMaps wm;
  e = make_window_maps(s, q, k, v, &wm);
  if (e != cudaSuccess) return e;
  const size_t wsb = window_state_bytes(s, w.PT);
  auto wstate = [&](int t0) -> void* { return W + w.wst + ((t0 / w.PT) & 1) * wsb; };
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_side_mu);  // one call's records and waits at a time
  Side& sd = g_side[dev];
  e = side_init(sd);
  if (e != cudaSuccess) return e;
  // the side stream starts after the work already on `st` (inputs, workspace)
  e = cudaEventRecord(sd.start, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(sd.st, sd.start, 0);
  if (e == cudaSuccess) e = launch_attn_window(s, wm, wstate(0), 0, std::min(w.PT, s.N), w.PT, sd.st, ctx);
  if (e == cudaSuccess) e = cudaEventRecord(sd.win, sd.st);
  if (e != cudaSuccess) return e;

  for (int t0 = 0; t0 < s.N; t0 += w.PT) {
    const int np = std::min(w.PT, s.N - t0);
    if (U > 0) {
      e = cudaMemsetAsync(cnt, 0, (size_t)U * 4, st);
      if (e != cudaSuccess) return e;
      const int grid = s.B * s.Hkv * ((np + PB - 1) / PB);
      const size_t hsmem = (size_t)s.C * sizeof(int);  // C <= 8192: at most 32 KB
      bucket_count_kernel<<<grid, 512, hsmem, st>>>(s, idx, t0, np, cnt, ctx);
      bucket_scan_kernel<<<1, 1024, 0, st>>>(U, cnt, off, ioff);
      bucket_scatter_kernel<<<grid, 512, hsmem, st>>>(s, idx, t0, np, off, ioff, cnt, ent, items);
      const long long nrows = (long long)s.B * s.Hkv * np;
      regroup_q_kernel<<<(unsigned)((nrows + 7) / 8), 256, 0, st>>>(s, (const __nv_bfloat16*)q, t0, np, w.PT, qg);
    }
    e = cudaStreamWaitEvent(st, sd.win, 0);  // window(t) done
    if (e != cudaSuccess) return e;
    if (U > 0) {
      attn_chunk_kernel<<<sms, THREADS, kSmemBytes, st>>>(s, tmk, tmv, ioff, items, ent, w.PT, qg, part, ctx);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    if (t0 + w.PT < s.N) {
      // window(t + 1) overwrites the state that fusion(t - 1), earlier on `st`, read
      e = cudaEventRecord(sd.next, st);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(sd.st, sd.next, 0);
      const int t1 = t0 + w.PT;
      if (e == cudaSuccess)
        e = launch_attn_window(s, wm, wstate(t1), t1, std::min(w.PT, s.N - t1), w.PT, sd.st, ctx);
      if (e == cudaSuccess) e = cudaEventRecord(sd.win, sd.st);
      if (e != cudaSuccess) return e;
    }
    e = launch_attn_fuse(s, idx, s_sel, part, wstate(t0), out, t0, np, w.PT, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace hils
