// Window attention and fusion of the chunk-major prefill (bf16, d = 128,
// S = 64, G = 4), on the tcgen05 tensor cores.
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method): position i attends the chunk-aligned window Win(i) (chunks
// cur - nw + 1 .. cur, causal inside cur) with exact softmax terms, and
//   out_i = (sum_c e^{s^_c} O_c + sum_{j in Win(i)} e^{s_j} v_j) / Z^_i,
//   Z^_i = sum_c e^{s^_c} + Z_swa,  Z_swa = sum_{j in Win(i)} e^{s_j}.
//
// attn_window_kernel: the window part.  Positions of one 32-aligned block lie
// in one chunk, so they share their window chunks; an item is such a block in
// one KV group, 32 positions x 4 heads = 128 query rows (row = 32 h + j), the
// MMA's M.  The window chunks are taken two at a time (adjacent chunks are
// one contiguous 128-key tile; an odd count pads with chunk cur + 1, whose
// keys the causal mask removes), so that each MMA instruction has N = 128
// keys for S and K = 128 keys for P V.  Two passes over the item's tiles:
//   pass 1: S_w = Q K_w^T (tcgen05, fp32 in TMEM), row maximum m;
//   pass 2: S_w again, P_w = e^{(s - m) scale} (<= 1) in bf16 over S's
//           columns, O += P_w V_w accumulated in TMEM, l = sum of P_w (fp32).
// Recomputing S (the tensor pipe is mostly idle here) keeps every weight at or
// below one without rescaling O in TMEM.  Measured at 128K: tiles of two
// chunks instead of one took the attention call from 20.3 to 19.8 ms (96
// instead of 160 MMA instructions per item of 8 chunks, from one issuing
// thread).  The item's (A, Z) = (O, l) relative
// to the reference exponent m go to the window state for the fusion kernel.
//
// CTA layout (one persistent CTA per SM, 320 threads, items dealt round-robin):
//   warp 0      TMA loads: the item's query rows (4 heads x 2 d-halves of 32
//               rows, 128-byte swizzle) and the window's K and V tiles
//               (4-stage ring of 32 KB tiles), in the order the MMA warp
//               consumes them
//   warp 1      tcgen05.mma issue (one thread)
//   warps 2-5   softmax, one row per thread (its TMEM lane)
//   warps 6-9   epilogue: O row -> window state
//
// attn_fuse_kernel: the fusion.  Per query-head row, with M = max(m', max_c s^_c)
// (m' = m scale in log2 units):
//   out = (A e^{m' - M} + sum_c e^{s^_c - M} O_c) / (Z e^{m' - M} + sum_c e^{s^_c - M}),
// O_c the partial records of attn_chunk.cu.  One warp per (sequence x KV
// group, position) reads each 1 KB record with two warp loads of 512
// contiguous bytes; measured on B200 at 128K it streams the records at about
// the measured HBM copy bandwidth.
//
// Every wait is bounded (status word + early return), see common.cuh.
#include <algorithm>

#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int D = 128, S = 64, G = 4;
constexpr int BPOS = 32;               // positions per item
constexpr int MR = BPOS * G;           // query rows per item (MMA M)
constexpr int TK = 2 * S;              // keys per tile: two adjacent window chunks
constexpr int NKV = 4;                 // K/V tile stages
constexpr uint32_t BOX = TK * 128;     // [128 keys x 64 d] bf16 (16 KB)
constexpr uint32_t QHALF = MR * 128;   // [128 rows x 64 d] bf16 (16 KB)
constexpr uint32_t QHEAD = BPOS * 128; // one head's 32 rows of a d-half (4 KB)
constexpr int THREADS = 10 * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t OCOL = 0;           // O of buffer ob at OCOL + 128 ob
constexpr uint32_t SCOL = 256;         // S / P of stage st at SCOL + 128 st
constexpr int KMAX = 64;

struct __align__(1024) SmemW {
  unsigned char q[2][2][QHALF];    // [buffer][d half][row][128 B]
  unsigned char kv[NKV][2][BOX];   // [stage][d half][key][128 B]
  uint64_t qfull[2], qempty[2], kvfull[NKV], kvempty[NKV];
  uint64_t sfull[2], pfull[2], sfree[2], ofull[2], ofree[2], done;
  uint32_t tmem;
};
constexpr size_t kSmemBytes = sizeof(SmemW) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

// item it of a tile: sequence x group bg, block of 32 positions from p0
struct WItem {
  int bg, p0, wc0, n;  // window chunks wc0 .. wc0 + n - 1 (the last is the block's own); n tiles of 2 chunks
};

__global__ void __launch_bounds__(THREADS, 1)
    attn_window_kernel(Shape s, const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, int t0, int np, int PT, float* __restrict__ wacc,
                       float* __restrict__ wmd, DevCtx ctx) {
  extern __shared__ unsigned char smem_raw[];
  SmemW& sm = *reinterpret_cast<SmemW*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nblk = (np + BPOS - 1) / BPOS;
  const int nitems = s.B * s.Hkv * nblk;
  const int bid = blockIdx.x, nb = gridDim.x;
  const int nmine = nitems > bid ? (nitems - 1 - bid) / nb + 1 : 0;
  const int pend = t0 + np;
  auto item_of = [&](int li) -> WItem {
    const int it = bid + li * nb;
    WItem r;
    r.bg = it / nblk;
    r.p0 = t0 + (it - r.bg * nblk) * BPOS;
    const int cur = r.p0 / S;
    r.wc0 = max(0, cur - s.nw + 1);
    r.n = (cur - r.wc0 + 2) / 2;  // tiles of two chunks; an odd count pads with chunk cur + 1 (all masked)
    return r;
  };

  if (tid == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.qfull[x], 1);
      mbar_init(&sm.qempty[x], 1);
      mbar_init(&sm.sfull[x], 1);
      mbar_init(&sm.pfull[x], 4);
      mbar_init(&sm.sfree[x], 1);
      mbar_init(&sm.ofull[x], 1);
      mbar_init(&sm.ofree[x], 4);
    }
    for (int x = 0; x < NKV; ++x) {
      mbar_init(&sm.kvfull[x], 1);
      mbar_init(&sm.kvempty[x], 1);
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
    // ------------------------------------------------------------ loads ----
    // per item: Q; pass 1: K_0 .. K_{n-1}; pass 2: K_0, then K_{w+1}, V_w
    // for each w (the MMA warp's order), V_{n-1} last
    if (lane == 0) {
      bool ok = true;
      int kt = 0, nq = 0;  // K/V tiles and query tiles issued
      if (nmine > 0) {
        prefetch_tmap(&tmq);
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
      }
      auto tile = [&](bool isv, int c, int bg) -> bool {
        const int x = kt % NKV;
        if (kt >= NKV && !mbar_wait(&sm.kvempty[x], ((kt / NKV) - 1) & 1, ctx)) return false;
        if (ctx.inject != 1) {  // host fault injection: no copy, the consumers' waits run out
          mbar_arrive_expect_tx(&sm.kvfull[x], 2 * BOX);
          tma_load_3d(sm.kv[x][0], isv ? &tmv : &tmk, 0, c * S, bg, &sm.kvfull[x]);
          tma_load_3d(sm.kv[x][1], isv ? &tmv : &tmk, 64, c * S, bg, &sm.kvfull[x]);
        }
        ++kt;
        return true;
      };
      for (int li = 0; li < nmine && ok; ++li) {
        const WItem im = item_of(li);
        const int qb = li & 1;
        if (li >= 2 && !mbar_wait(&sm.qempty[qb], ((li >> 1) - 1) & 1, ctx)) {
          ok = false;
          break;
        }
        const int b = im.bg / s.Hkv, g = im.bg - b * s.Hkv;
        if (ctx.inject != 1) {
          mbar_arrive_expect_tx(&sm.qfull[qb], 2 * QHALF);
          for (int h = 0; h < G; ++h)
            for (int hf = 0; hf < 2; ++hf)
              tma_load_3d(sm.q[qb][hf] + h * QHEAD, &tmq, 64 * hf, im.p0, b * s.Hq + g * G + h, &sm.qfull[qb]);
          ++nq;
        }
        for (int w = 0; w < im.n && ok; ++w) ok = tile(false, im.wc0 + 2 * w, im.bg);
        if (ok) ok = tile(false, im.wc0, im.bg);
        for (int w = 0; w < im.n && ok; ++w) {
          if (w + 1 < im.n) ok = tile(false, im.wc0 + 2 * (w + 1), im.bg);
          if (ok) ok = tile(true, im.wc0 + 2 * w, im.bg);
        }
      }
      // the copies issued last land before the CTA exits, whichever role gave
      // up first (their phases completed long ago on the normal path)
      if (ctx.inject != 1)
        for (int j = std::max(0, kt - NKV); j < kt; ++j) mbar_wait(&sm.kvfull[j % NKV], (j / NKV) & 1, ctx);
      for (int j = std::max(0, nq - 2); j < nq; ++j) mbar_wait(&sm.qfull[j & 1], (j >> 1) & 1, ctx);
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issue ----
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(MR, TK);
      const uint32_t idO = idesc_bf16_f32(MR, D) | (1u << 16);  // B (V) is MN-major
      int kt = 0, u = 0;            // K/V tiles consumed, S-stage uses
      int kind[2] = {0, 0};         // last use of each S stage: 1 = pass 1, 2 = pass 2
      int n2[2] = {0, 0};           // pass-2 uses of each stage (commits on sfree)
      // S = Q K^T into stage u % 2 once its previous use is over: a pass-1 use
      // ends when the softmax has read S (pfull), a pass-2 use when the O MMA
      // has read P (sfree)
      auto issue_s = [&](int qb, int pass, int& st_out, int& u_out) -> bool {
        const int st = u & 1;
        if (kind[st] == 1 && !mbar_wait(&sm.pfull[st], ((u - 2) >> 1) & 1, ctx)) return false;
        if (kind[st] == 2 && !mbar_wait(&sm.sfree[st], (n2[st] - 1) & 1, ctx)) return false;
        const int x = kt % NKV;
        if (!mbar_wait(&sm.kvfull[x], (kt / NKV) & 1, ctx)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = sdesc_k_sw128(smem_u32(sm.q[qb][kk >> 2]) + (kk & 3) * 32);
          const uint64_t bd = sdesc_k_sw128(smem_u32(sm.kv[x][kk >> 2]) + (kk & 3) * 32);
          mma_ss(tmem + SCOL + 128 * st, ad, bd, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&sm.sfull[st]);
        tc_commit(&sm.kvempty[x]);
        kind[st] = pass;
        st_out = st;
        u_out = u;
        ++kt;
        ++u;
        return true;
      };
      // O (+)= P V once the softmax has written P of use uw into stage st
      auto issue_o = [&](int st, int uw, int ob, bool first) -> bool {
        if (!mbar_wait(&sm.pfull[st], (uw >> 1) & 1, ctx)) return false;
        const int x = kt % NKV;
        if (!mbar_wait(&sm.kvfull[x], (kt / NKV) & 1, ctx)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < TK / 16; ++kk) {
          const uint64_t bd = sdesc_mn_sw128(smem_u32(sm.kv[x][0]) + kk * 2048, BOX, 1024);
          mma_ts(tmem + OCOL + 128 * ob, tmem + SCOL + 128 * st + 8 * kk, bd, idO, (first && kk == 0) ? 0u : 1u);
        }
        tc_commit(&sm.sfree[st]);
        ++n2[st];
        tc_commit(&sm.kvempty[x]);
        ++kt;
        return true;
      };
      bool ok = true;
      for (int li = 0; li < nmine && ok; ++li) {
        const WItem im = item_of(li);
        const int qb = li & 1, ob = li & 1;
        ok = mbar_wait(&sm.qfull[qb], (li >> 1) & 1, ctx);
        int st = 0, uw = 0, st1 = 0, u1 = 0;
        for (int w = 0; w < im.n && ok; ++w) ok = issue_s(qb, 1, st, uw);
        if (ok && li >= 2) ok = mbar_wait(&sm.ofree[ob], ((li >> 1) - 1) & 1, ctx);
        if (ok) ok = issue_s(qb, 2, st, uw);
        for (int w = 0; w < im.n && ok; ++w) {
          if (w + 1 < im.n) ok = issue_s(qb, 2, st1, u1);
          if (ok) ok = issue_o(st, uw, ob, w == 0);
          st = st1;
          uw = u1;
        }
        if (ok) {
          tc_commit(&sm.qempty[qb]);
          tc_commit(&sm.ofull[ob]);
        }
      }
      // every MMA issued above has completed before the columns are released
      tc_commit(&sm.done);
      mbar_wait(&sm.done, 0, ctx);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ---------------------------------------------------------- softmax ----
    // thread = TMEM lane = row 32 h + j: head h = warp % 4, position p0 + j
    const int h = warp & 3;
    const uint32_t lrow = (uint32_t)(32 * h) << 16;
    const float sl2 = s.scale * kLog2e;
    int u = 0;
    bool ok = true;
    for (int li = 0; li < nmine && ok; ++li) {
      const WItem im = item_of(li);
      const int p = im.p0 + lane;
      float m = -INFINITY, l = 0.f, base = 0.f;
      for (int pass = 1; pass <= 2 && ok; ++pass) {
        if (pass == 2) base = m * sl2;
        for (int w = 0; w < im.n; ++w) {
          const int st = u & 1;
          // keys of this tile at or before p (at least one: its first chunk is <= p's)
          const int lim = p - (im.wc0 + 2 * w) * S + 1;
          ok = mbar_wait(&sm.sfull[st], (u >> 1) & 1, ctx);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
          float z = 0.f;
#pragma unroll
          for (int hk = 0; hk < 2; ++hk) {  // keys 64 hk .. 64 hk + 63
            uint32_t r0[32], r1[32];
            tmem_ld32(tmem + lrow + SCOL + 128 * st + 64 * hk, r0);
            tmem_ld32(tmem + lrow + SCOL + 128 * st + 64 * hk + 32, r1);
            tmem_wait_ld();
            if (lim < 64 * hk + 64) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if (64 * hk + j >= lim) r0[j] = __float_as_uint(-INFINITY);
                if (64 * hk + j + 32 >= lim) r1[j] = __float_as_uint(-INFINITY);
              }
            }
            if (pass == 1) {
              float mx = m;
#pragma unroll
              for (int j = 0; j < 32; ++j) mx = fmaxf(mx, fmaxf(__uint_as_float(r0[j]), __uint_as_float(r1[j])));
              m = mx;
            } else {
              uint32_t pw[16];
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const float e0 = exp2f(fmaf(__uint_as_float(r0[2 * c]), sl2, -base));
                const float e1 = exp2f(fmaf(__uint_as_float(r0[2 * c + 1]), sl2, -base));
                z += e0 + e1;
                pw[c] = pack_bf16x2(e0, e1);
              }
              tmem_st16(tmem + lrow + SCOL + 128 * st + 32 * hk, pw);
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const float e0 = exp2f(fmaf(__uint_as_float(r1[2 * c]), sl2, -base));
                const float e1 = exp2f(fmaf(__uint_as_float(r1[2 * c + 1]), sl2, -base));
                z += e0 + e1;
                pw[c] = pack_bf16x2(e0, e1);
              }
              tmem_st16(tmem + lrow + SCOL + 128 * st + 32 * hk + 16, pw);
            }
          }
          if (pass == 2) {
            tmem_wait_st();
            l += z;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.pfull[st]);
          ++u;
        }
      }
      if (ok && p < pend) {
        const long long rowb = (long long)im.bg * PT + (p - t0);
        *reinterpret_cast<float2*>(wmd + (rowb * G + h) * 2) = make_float2(base, l);
      }
    }
  } else {
    // --------------------------------------------------------- epilogue ----
    // O row (d = 0..127) -> wacc[bg][p - t0][cls][h][i], d = 8 i + cls
    const int h = warp & 3;
    const uint32_t lrow = (uint32_t)(32 * h) << 16;
    for (int li = 0; li < nmine; ++li) {
      const WItem im = item_of(li);
      const int ob = li & 1, p = im.p0 + lane;
      const bool ok = mbar_wait(&sm.ofull[ob], (li >> 1) & 1, ctx);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      float* dst = wacc + ((long long)im.bg * PT + (p - t0)) * (8 * G * 16) + h * 16;
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) {
        uint32_t v[32];
        tmem_ld32(tmem + lrow + OCOL + 128 * ob + 32 * qd, v);
        tmem_wait_ld();
        if (p < pend) {
#pragma unroll
          for (int cls = 0; cls < 8; ++cls)
            *reinterpret_cast<float4*>(dst + cls * (G * 16) + 4 * qd) =
                make_float4(__uint_as_float(v[cls]), __uint_as_float(v[cls + 8]), __uint_as_float(v[cls + 16]),
                            __uint_as_float(v[cls + 24]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.ofree[ob]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// ---------------------------------------------------------------- fusion ----
// One warp per (sequence x KV group, position); lane l = 4 cls + h owns head
// h's values d = 8 i + cls (i = 0..15).  A record (1 KB, [unit][head][32 B],
// attn_chunk.cu) is read by two warp loads of 512 contiguous bytes: piece
// (h2, cls) of head h, 16 bytes in unit 4 h2 + cls / 2 at half cls % 2, holds
// d = 64 h2 + 32 a + cls + 8 t at element e = 4 a + t, i.e. i = 8 h2 + e.
// Slots are read 4 at a time, predicated on their weight, so that their HBM
// round trips overlap.  The list is checked with the bucketing's acceptance
// rule, so both agree on every pair.
constexpr int FW = 8;  // warps per fusion block

__global__ void __launch_bounds__(FW * 32) attn_fuse_kernel(Shape s, const int32_t* __restrict__ idx,
                                                           const float* __restrict__ s_sel,
                                                           const __nv_bfloat16* __restrict__ part,
                                                           const float* __restrict__ wacc,
                                                           const float* __restrict__ wmd,
                                                           __nv_bfloat16* __restrict__ out, int t0, int np, int PT) {
  __shared__ float wsm[FW][KMAX][G];
  __shared__ __align__(16) __nv_bfloat16 osm[FW][G][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long wid = (long long)blockIdx.x * FW + warp;
  if (wid >= (long long)s.B * s.Hkv * np) return;  // whole warps only; no block barrier below
  const int bg = (int)(wid / np), pl = (int)(wid - (long long)bg * np);
  const int b = bg / s.Hkv, g = bg - b * s.Hkv, p = t0 + pl, K = s.K;
  const int cls = lane >> 2, h = lane & 3;
  const int32_t* L = idx + ((long long)bg * s.N + p) * K;
  int la = lane < K ? __ldg(L + lane) : -1;
  int lb = lane + 32 < K ? __ldg(L + lane + 32) : -1;
  bool bad;  // reported by the bucketing, which applies the same rule
  accept_list_warp(la, lb, K, max(0, p / S - s.nw + 1), bad);
  const long long rowb = (long long)bg * PT + pl;
  float fw = 0.f, zden = 1.f;  // this lane's head: window factor e^{m' - M}, denominator
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const float* sr = s_sel + (((long long)b * s.Hq + g * G + hh) * s.N + p) * K;
    const float xa = la >= 0 ? __ldg(sr + lane) * kLog2e : -INFINITY;
    const float xb = lb >= 0 ? __ldg(sr + lane + 32) * kLog2e : -INFINITY;
    float mx = fmaxf(xa, xb);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float2 md = __ldg(reinterpret_cast<const float2*>(wmd + (rowb * G + hh) * 2));
    const float M = fmaxf(md.x, mx);
    const float wa = xa == -INFINITY ? 0.f : exp2f(xa - M);
    const float wb = xb == -INFINITY ? 0.f : exp2f(xb - M);
    if (lane < K) wsm[warp][lane][hh] = wa;
    if (lane + 32 < K) wsm[warp][lane + 32][hh] = wb;
    float z = wa + wb;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float f = exp2f(md.x - M);
    if (hh == h) {
      fw = f;
      zden = md.y * f + z;
    }
  }
  __syncwarp();
  float acc[16];
  {
    const float4* wa = reinterpret_cast<const float4*>(wacc + (rowb * 8 + cls) * (G * 16) + h * 16);
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float4 v = __ldg(wa + x);
      acc[4 * x + 0] = v.x * fw;
      acc[4 * x + 1] = v.y * fw;
      acc[4 * x + 2] = v.z * fw;
      acc[4 * x + 3] = v.w * fw;
    }
  }
  const __nv_bfloat16* rec = part + rowb * K * (G * D) + (cls >> 1) * (G * 16) + h * 16 + (cls & 1) * 8;
  for (int k0 = 0; k0 < K; k0 += 4) {
    uint4 u[4][2];
    float wk[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = k0 + j;
      const float w = k < K ? wsm[warp][k][h] : 0.f;
      wk[j] = w;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (w > 0.f) x = __ldg(reinterpret_cast<const uint4*>(rec + (long long)k * (G * D) + h2 * (4 * G * 16)));
        u[j][h2] = x;
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const uint32_t ww[4] = {u[j][h2].x, u[j][h2].y, u[j][h2].z, u[j][h2].w};
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) {
          const float2 f = bf16x2_to_f32x2(ww[q2]);
          acc[8 * h2 + 2 * q2] = fmaf(wk[j], f.x, acc[8 * h2 + 2 * q2]);
          acc[8 * h2 + 2 * q2 + 1] = fmaf(wk[j], f.y, acc[8 * h2 + 2 * q2 + 1]);
        }
      }
  }
  const float inv = 1.f / zden;
#pragma unroll
  for (int i = 0; i < 16; ++i) osm[warp][h][8 * i + cls] = __float2bfloat16_rn(acc[i] * inv);
  __syncwarp();
  {
    const int hh = lane >> 3, x = lane & 7;
    const uint4* src = reinterpret_cast<const uint4*>(&osm[warp][hh][16 * x]);
    uint4* dst = reinterpret_cast<uint4*>(out + (((long long)b * s.Hq + g * G + hh) * s.N + p) * D + 16 * x);
    dst[0] = src[0];
    dst[1] = src[1];
  }
}

}  // namespace

size_t window_state_bytes(const Shape& s, int PT) { return (size_t)s.B * s.Hkv * PT * G * (8 * 16 + 2) * 4; }

cudaError_t make_window_maps(const Shape& s, const void* q, const void* k, const void* v, WindowMaps* m) {
  if (s.d != D || s.S != S || s.G != G || s.K > KMAX || s.nw < 1) return cudaErrorNotSupported;
  const uint64_t qdims[3] = {(uint64_t)D, (uint64_t)s.N, (uint64_t)s.B * s.Hq};
  const uint64_t kdims[3] = {(uint64_t)D, (uint64_t)s.N, (uint64_t)s.B * s.Hkv};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)s.N * D * 2};
  const uint32_t qbox[3] = {64, (uint32_t)BPOS, 1};
  const uint32_t kbox[3] = {64, (uint32_t)TK, 1};
  cudaError_t e = make_tmap_bf16(&m->q, q, 3, qdims, strides, qbox, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&m->k, k, 3, kdims, strides, kbox, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  return make_tmap_bf16(&m->v, v, 3, kdims, strides, kbox, CU_TENSOR_MAP_SWIZZLE_128B);
}

// window state: accumulators [B Hkv][PT][8][G][16], then (m', l) [B Hkv][PT][G][2]
static float* window_md(const Shape& s, void* wstate, int PT) {
  return (float*)wstate + (size_t)s.B * s.Hkv * PT * 8 * G * 16;
}

cudaError_t launch_attn_window(const Shape& s, const WindowMaps& m, void* wstate, int t0, int np, int PT,
                               cudaStream_t st, const DevCtx& ctx) {
  if (t0 % BPOS || np < 1 || np > PT || !wstate) return cudaErrorInvalidValue;
  cudaError_t e = ensure_dynamic_smem((const void*)attn_window_kernel, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int nitems = s.B * s.Hkv * ((np + BPOS - 1) / BPOS);
  const int grid = std::min(nitems, device_sm_count());
  attn_window_kernel<<<grid, THREADS, kSmemBytes, st>>>(s, m.q, m.k, m.v, t0, np, PT, (float*)wstate,
                                                        window_md(s, wstate, PT), ctx);
  return cudaGetLastError();
}

cudaError_t launch_attn_fuse(const Shape& s, const int32_t* idx, const float* s_sel, const void* part,
                             const void* wstate, void* out, int t0, int np, int PT, cudaStream_t st) {
  if (np < 1 || np > PT || !part || !wstate) return cudaErrorInvalidValue;
  const long long rows = (long long)s.B * s.Hkv * np;
  attn_fuse_kernel<<<(unsigned)((rows + FW - 1) / FW), FW * 32, 0, st>>>(
      s, idx, s_sel, (const __nv_bfloat16*)part, (const float*)wstate, window_md(s, (void*)wstate, PT),
      (__nv_bfloat16*)out, t0, np, PT);
  return cudaGetLastError();
}

}  // namespace hils
