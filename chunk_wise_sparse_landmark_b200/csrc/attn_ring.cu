// Hierarchical-softmax sparse attention, bf16 prefill (d = 128, S = 64, G = 4).
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method): each selected chunk is attended with its own softmax, the chunk
// outputs are weighted by exp(s^_{i,c}) / Z^_i and the chunk-aligned window by
// Z_swa / Z^_i, Z^_i = sum_c exp(s^_{i,c}) + Z_swa.  The section's hardware
// paragraph groups adjacent queries and attends the union of their chunks;
// here a CTA groups 14 adjacent positions of one GQA group (56 query-head
// rows) and streams the union of their chunks once.
//
// Why this shape.  Moving 64-key chunk tiles from L2 to the SMs is what
// bounds this operation.  Even when positions pick their top-K chunks
// independently, P positions choosing K of n candidates cover only
// n (1 - (1 - K/n)^P) distinct chunks, and they share their window chunks.
// One producer warp streams the union -- the block's selections below its
// first window chunk (a bitmap, in chunk order), then every chunk from there
// to the last position's chunk -- as separate K and V tiles (16 KB each,
// 128-byte swizzle, rows past the sequence read as zero) through a 6-slot
// shared-memory ring filled by the tensor-memory accelerator.  7 consumer
// warps, one per pair of positions (8 rows), each walk only their own chunks
// (the two selection lists merged, then their window) in stream order.  A
// slot is released by the warps that use its tile: the producer knows each
// tile's user count (taken from the walks before streaming starts) and
// arrives for the other warps itself, so a slot is never held by warps that
// skip it.  Two such CTAs share an SM (256 threads, 128 registers each, about
// 100 KB of shared memory): measured on B200, two independent rings per SM
// beat one CTA of 15 consumer warps with a 13-slot ring (97.5 vs 101.0 ms at
// 128K), because one stream's stalls no longer idle the whole SM.  A block
// may straddle two chunks, so each warp keeps its own window range.
//
// Ring protocol.  The items are the chunks' K and V tiles in stream order,
// except that chunk r's V tile follows chunk r + DV's K tile: it is needed
// only after the chunk's S^T and softmax, and holding it in a slot meanwhile
// costs ring capacity (measured: 96.2 -> 91.1 ms at 128K for DV = 1).  Each
// consumer then meets at most DV of its items out of stream order, which is
// deadlock-free while NSI > DV: the producer issues in stream order, and an
// item's slot is only reused after every earlier item in that slot was
// released by its users.  Item k lives in slot k % NSI; its round k / NSI is
// published in round_[slot] once the slot's previous round has been
// released, and only then does a consumer wait on the slot's full barrier
// with that round's parity (a consumer may run many items ahead of the
// producer, so the parity alone would be ambiguous).
//
//   S^T (64 keys x 8 rows)   = K_c (keys x d)  . Q^T (d x rows)
//   O^T (128 d x 8 rows)    += V_c^T (d x keys) . P^T (keys x rows)
//
// bf16 mma.sync m16n8k16 with fp32 accumulation, A fragments by ldmatrix
// (K tile as stored, V tile transposed), P^T by an in-register transpose of
// the S^T accumulator (movmatrix).
//
// Row state (per query-head row): m2 = reference exponent (log2 units, >= all
// exponents used so far), den = sum of weights, acc = weighted values.
// Selected chunk: P_j = e^{s_j - mu}/Z_c * e^{s^ - m}, den += e^{s^ - m}.
// Window chunk: P_j = e^{s_j - m}, den += sum_j P_j; m is raised (acc and den
// rescaled) when a window logit exceeds it.  out = acc / den.
#include <climits>

#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int D = 128, S = 64, G = 4;
constexpr int CW = 7;                   // consumer warps, one per position pair
constexpr int BP = 2 * CW;              // positions per CTA
constexpr int THREADS = (CW + 1) * 32;  // + producer warp
constexpr int NSI = 6;                  // ring slots (16 KB each)
constexpr uint32_t BOX = 64 * 128;      // [64 keys x 64 d] bf16, 128-byte rows
constexpr uint32_t ITEM = 2 * BOX;      // the K or V tile of one chunk
constexpr int KMAX = 64;
constexpr int MAXC = 8192;              // candidate chunks covered by the bitmap
constexpr int MAXW = MAXC / 32;
constexpr int MAXI = 2048;              // stream chunks per CTA (>= BP * KMAX + window)
constexpr int MSL = 3;                  // partial-record slots loaded at a time

struct __align__(1024) SmemR {
  unsigned char slot[NSI][2][BOX];
  uint32_t bits[MAXW];          // the block's selections below lo
  uint32_t pre[MAXW];           // exclusive prefix of popc(bits)
  uint32_t users[MAXI / 4];     // warps using each stream chunk (bytes)
  int round_[NSI];
  uint64_t full[NSI], empty[NSI];
  int nb;                       // selections below lo = stream chunks from the bitmap
};

// shared-memory fragment loads; the "memory" clobber keeps them ahead of the
// barrier arrive that hands their slot back to the copy engine
HILS_DI void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
HILS_DI void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
HILS_DI uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
HILS_DI void mbar_arrive_cnt(uint64_t* bar, uint32_t cnt) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
               "r"(cnt)
               : "memory");
}
// byte address of 16-byte unit `unit` (0..7) of row `row` in a 128-byte-swizzled box
HILS_DI uint32_t swz(uint32_t box, int row, int unit) { return box + row * 128 + ((unit ^ (row & 7)) << 4); }

// Ring item numbers of stream chunk r's K and V tiles (n chunks): K_0 .. K_{DV-1},
// then K_{r+DV}, V_r alternating, then the last DV V tiles.
constexpr int DV = 1;
static_assert(NSI > DV, "the delayed V tiles need more slots than the delay");
HILS_DI int item_k(int r) { return r < DV ? r : 2 * r - DV; }
HILS_DI int item_v(int r, int n) { return r <= n - 1 - DV ? DV + 2 * r + 1 : n + r; }

// A warp's chunks in stream order: the merged selection lists, then its window.
struct Walk {
  int cu0 = 0, cu1 = 0, w = 0;
  int c = 0;  // current chunk, INT_MAX at the end
  bool win = false, part0 = false, part1 = false;
  int slot0 = 0, slot1 = 0;  // positions in the two lists (s^ lookup)
};

__global__ void __launch_bounds__(THREADS, 2)
    attn_ring_kernel(Shape s, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                     const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ idx,
                     const float* __restrict__ s_sel, __nv_bfloat16* __restrict__ out,
                     DevCtx ctx) {
  extern __shared__ unsigned char smem_raw[];
  SmemR& sm = *reinterpret_cast<SmemR*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y, b = blockIdx.z;
  const int bg = b * s.Hkv + g;
  const int i0 = blockIdx.x * BP;
  const int nend = s.N;
  const int K = s.K;
  // stream: selected chunks below lo (bitmap, ascending), then every chunk lo..hi
  const int lo = max(0, i0 / S - s.nw + 1);    // first window chunk of the block
  const int hi = (min(i0 + BP, nend) - 1) / S;  // chunk of the block's last position
  const int nwords = (lo + 31) >> 5;

  for (int x = tid; x < nwords; x += THREADS) sm.bits[x] = 0u;
  for (int x = tid; x < MAXI / 4; x += THREADS) sm.users[x] = 0u;
  if (tid == 0) {
    for (int x = 0; x < NSI; ++x) {
      mbar_init(&sm.full[x], 1);
      mbar_init(&sm.empty[x], CW);
      sm.round_[x] = -1;
    }
    fence_barrier_init();
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
  }
  __syncthreads();

  // consumer state (warp < CW): positions p0, p0 + 1 (same chunk: p0 is even)
  const int p0 = i0 + 2 * warp;
  const bool valid0 = warp < CW && p0 < nend;
  const bool valid1 = warp < CW && p0 + 1 < nend;
  const int cur = p0 / S;
  const int ncand = max(0, cur - s.nw + 1);
  const int wc0 = ncand;  // this warp's window chunks wc0..cur
  int l0a = -1, l0b = -1, l1a = -1, l1b = -1;  // lane j: list entries j and j + 32
  if (warp < CW) {
    const int32_t* L0 = idx + ((long long)bg * s.N + p0) * K;
    if (valid0) {
      l0a = lane < K ? __ldg(L0 + lane) : -1;
      l0b = lane + 32 < K ? __ldg(L0 + lane + 32) : -1;
    }
    if (valid1) {
      l1a = lane < K ? __ldg(L0 + K + lane) : -1;
      l1b = lane + 32 < K ? __ldg(L0 + K + lane + 32) : -1;
    }
    // entries that break the list form (ascending candidates, then -1) are
    // dropped and reported; the chunk-major bucketing drops the same ones
    bool bad0, bad1;
    accept_list_warp(l0a, l0b, K, ncand, bad0);
    accept_list_warp(l1a, l1b, K, ncand, bad1);
    if ((bad0 || bad1) && lane == 0) raise_status(ctx, kStatusBadIndex);
  }
  if (warp < CW) {
    if (l0a >= 0 && l0a < lo) atomicOr(&sm.bits[l0a >> 5], 1u << (l0a & 31));
    if (l0b >= 0 && l0b < lo) atomicOr(&sm.bits[l0b >> 5], 1u << (l0b & 31));
    if (l1a >= 0 && l1a < lo) atomicOr(&sm.bits[l1a >> 5], 1u << (l1a & 31));
    if (l1b >= 0 && l1b < lo) atomicOr(&sm.bits[l1b >> 5], 1u << (l1b & 31));
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive prefix of the bitmap's popcounts
    int run = 0;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
      const int w = w0 + lane;
      const int cnt = w < nwords ? __popc(sm.bits[w]) : 0;
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      if (w < nwords) sm.pre[w] = run + incl - cnt;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) sm.nb = run;
  }
  __syncthreads();
  const int nb = sm.nb;
  const int nchunks = nb + (hi - lo + 1);
  auto rank = [&](int c) -> int {
    if (c >= lo) return nb + (c - lo);
    const int w = c >> 5;
    return (int)sm.pre[w] + __popc(sm.bits[w] & ((1u << (c & 31)) - 1u));
  };

  // list entry `cu` (warp-uniform), -1 past the list
  auto entry = [&](int la, int lb, int cu) -> int {
    const int v = __shfl_sync(0xffffffffu, cu < 32 ? la : lb, cu & 31);
    return cu < K ? v : -1;
  };
  // the accepted entries of the two lists (dropped ones left -1 holes)
  const uint64_t vm0 = (uint64_t)__ballot_sync(0xffffffffu, l0a >= 0) |
                       ((uint64_t)__ballot_sync(0xffffffffu, l0b >= 0) << 32);
  const uint64_t vm1 = (uint64_t)__ballot_sync(0xffffffffu, l1a >= 0) |
                       ((uint64_t)__ballot_sync(0xffffffffu, l1b >= 0) << 32);
  // the first accepted entry at or after slot cu: its chunk (INT_MAX if none) and slot
  auto next_at = [&](int la, int lb, uint64_t vm, int cu, int& x) -> int {
    const uint64_t rest = cu < 64 ? (vm & (~0ull << cu)) : 0ull;
    x = rest ? __ffsll((long long)rest) - 1 : 0;
    const int v = __shfl_sync(0xffffffffu, x < 32 ? la : lb, x & 31);
    return rest ? v : INT_MAX;
  };
  auto step = [&](Walk& wk) {
    int x0, x1;
    const int a0 = next_at(l0a, l0b, vm0, wk.cu0, x0), a1 = next_at(l1a, l1b, vm1, wk.cu1, x1);
    if (a0 != INT_MAX || a1 != INT_MAX) {
      wk.c = min(a0, a1);
      wk.win = false;
      wk.part0 = a0 == wk.c;
      wk.part1 = a1 == wk.c;
      wk.slot0 = x0;
      wk.slot1 = x1;
      if (wk.part0) wk.cu0 = x0 + 1;
      if (wk.part1) wk.cu1 = x1 + 1;
    } else if (valid0 && wc0 + wk.w <= cur) {
      wk.c = wc0 + wk.w++;
      wk.win = true;
      wk.part0 = true;
      wk.part1 = valid1;
      wk.slot0 = wk.slot1 = 0;
    } else {
      wk.c = INT_MAX;
    }
  };
  if (warp < CW) {
    // user counts of the stream chunks
    Walk wk;
    for (step(wk); wk.c != INT_MAX; step(wk)) {
      const int r = rank(wk.c);
      if (lane == 0) atomicAdd(&sm.users[r >> 2], 1u << (8 * (r & 3)));
    }
  }
  __syncthreads();

  if (warp == CW) {
    // ---------------------------------------------------------- producer ----
    if (lane == 0) {
      bool ok = true;
      int k = 0;  // items issued
      int w = 0;
      uint32_t m = nwords > 0 ? sm.bits[0] : 0u;
      auto chunk_at = [&](int r) -> int {  // stream chunks, taken in order
        if (r >= nb) return lo + (r - nb);
        while (m == 0u) m = sm.bits[++w];
        const int c = 32 * w + __ffs(m) - 1;
        m &= m - 1u;
        return c;
      };
      auto users_at = [&](int r) -> int { return (int)((sm.users[r >> 2] >> (8 * (r & 3))) & 0xFFu); };
      auto put = [&](bool is_v, int c, int users) {
        const int x = k % NSI, mr = k / NSI;
        if (mr > 0) ok = mbar_wait(&sm.empty[x], (mr - 1) & 1, ctx);
        if (!ok) return;
        *reinterpret_cast<volatile int*>(&sm.round_[x]) = mr;
        if (ctx.inject != 1) {
          const CUtensorMap* tm = is_v ? &tmv : &tmk;
          mbar_arrive_expect_tx(&sm.full[x], ITEM);
          tma_load_3d(sm.slot[x][0], tm, 0, c * S, bg, &sm.full[x]);
          tma_load_3d(sm.slot[x][1], tm, 64, c * S, bg, &sm.full[x]);
        }
        // the warps that do not use this tile are counted as done with it
        if (users < CW) mbar_arrive_cnt(&sm.empty[x], (uint32_t)(CW - users));
        ++k;
      };
      // the last DV + 1 chunks (pc[DV] = the newest), a shift register with
      // static indices so that it stays in registers
      int pc[DV + 1], pu[DV + 1];
#pragma unroll
      for (int j = 0; j <= DV; ++j) pc[j] = pu[j] = 0;
      for (int r = 0; r < nchunks && ok; ++r) {
        const int c = chunk_at(r), u = users_at(r);
        put(false, c, u);
#pragma unroll
        for (int j = 0; j < DV; ++j) {
          pc[j] = pc[j + 1];
          pu[j] = pu[j + 1];
        }
        pc[DV] = c;
        pu[DV] = u;
        if (ok && r >= DV) put(true, pc[0], pu[0]);  // V tile of chunk r - DV
      }
      // V tiles of the last DV chunks (chunk n - 1 - DV + j sits at pc[j])
#pragma unroll
      for (int j = 1; j <= DV; ++j)
        if (ok && nchunks - 1 - DV + j >= 0) put(true, pc[j], pu[j]);
      // copies still in flight (only after a timeout) land before the CTA exits
      if (!ok && ctx.inject != 1)
        for (int j = max(0, k - NSI); j < k; ++j) mbar_wait(&sm.full[j % NSI], (j / NSI) & 1, ctx);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- consumers ---
    const int gq = lane >> 2, c4 = lane & 3;  // fragment coordinates
    // Q^T fragments of the 8 rows (row gq: position p0 + gq/4, head gq%4), k-step ks:
    // b0 = d 16ks + 2c4 (+1), b1 = d 16ks + 8 + 2c4 (+1)
    uint32_t qf[8][2];
    {
      const bool okq = (gq >> 2) == 0 ? valid0 : valid1;
      const __nv_bfloat16* qr = q + (((long long)b * s.Hq + g * G + (gq & 3)) * s.N + p0 + (gq >> 2)) * D;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        qf[ks][0] = okq ? __ldg(reinterpret_cast<const uint32_t*>(qr + 16 * ks + 2 * c4)) : 0u;
        qf[ks][1] = okq ? __ldg(reinterpret_cast<const uint32_t*>(qr + 16 * ks + 8 + 2 * c4)) : 0u;
      }
    }
    // this thread's two rows (columns of S^T / O^T): position my_q, heads my_h, my_h + 1
    const int my_q = c4 >> 1;
    const int my_h = 2 * (c4 & 1);
    const int my_pos = p0 + my_q;
    const bool my_valid = my_q == 0 ? valid0 : valid1;
    const float* ss0 = s_sel + (((long long)b * s.Hq + g * G + my_h) * s.N + my_pos) * K;
    const long long sstride = (long long)s.N * K;  // next head
    float m2[2], den[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = -INFINITY;
      if (my_valid)
        for (int x = 0; x < K; ++x) mx = fmaxf(mx, __ldg(ss0 + r * sstride + x));
      m2[r] = mx * kLog2e;
    }
    const float sl2 = s.scale * kLog2e;
    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    const int mi = lane >> 3, rr = lane & 7;
    bool ok = true;
    // wait for ring item k: its round is published, then its copy has landed
    auto acquire = [&](int k) -> bool {
      const int x = k % NSI, m = k / NSI;
      bool okw = true;
      if (*reinterpret_cast<volatile int*>(&sm.round_[x]) != m) {
        const long long t0 = clock64();
        while (*reinterpret_cast<volatile int*>(&sm.round_[x]) != m) {
          if (clock64() - t0 > ctx.wait_budget) {
            raise_status(ctx, kStatusTimeout);
            okw = false;
            break;
          }
          __nanosleep(64);
        }
      }
      if (okw) okw = mbar_wait(&sm.full[x], m & 1, ctx);
      return __all_sync(0xffffffffu, okw);
    };

    Walk wk;
    for (step(wk); wk.c != INT_MAX; step(wk)) {
      const int c = wk.c;
      const bool win = wk.win;
      const bool my_part = my_valid && (my_q == 0 ? wk.part0 : wk.part1);
      float a2[2] = {-INFINITY, -INFINITY};
      if (!win && my_part) {
        const int slot_me = my_q == 0 ? wk.slot0 : wk.slot1;
        a2[0] = __ldg(ss0 + slot_me) * kLog2e;
        a2[1] = __ldg(ss0 + sstride + slot_me) * kLog2e;
      }
      const int rk = rank(c);
      const int kit = item_k(rk), vit = item_v(rk, nchunks);
      // ---- K tile: S^T = K_c Q^T
      if (!acquire(kit)) {
        ok = false;
        break;
      }
      const uint32_t kb = smem_u32(sm.slot[kit % NSI][0]);
      float sc[4][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) sc[mt][0] = sc[mt][1] = sc[mt][2] = sc[mt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t box = kb + (ks >> 2) * BOX;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          uint32_t a[4];
          ldsm_x4(a, swz(box, 16 * mt + rr + 8 * (mi & 1), 2 * (ks & 3) + (mi >> 1)));
          mma_bf16_16816(sc[mt], a, qf[ks][0], qf[ks][1]);
        }
      }
      __syncwarp();
      fence_proxy_async_shared();
      if (lane == 0) mbar_arrive(&sm.empty[kit % NSI]);
      // ---- weights; this thread holds keys 16mt+gq (+8) of rows 2c4, 2c4+1
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float mx = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int key = 16 * mt + gq + 8 * hh;
            float tt = sc[mt][2 * hh + r] * sl2;
            if (!my_part || (win && c * S + key > my_pos)) tt = -INFINITY;
            sc[mt][2 * hh + r] = tt;
            mx = fmaxf(mx, tt);
          }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
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
          for (int hh = 0; hh < 2; ++hh) {
            const float tt = sc[mt][2 * hh + r];
            const float p = (my_part && tt != -INFINITY) ? exp2f(tt - base) : 0.f;
            sc[mt][2 * hh + r] = p;
            z += p;
          }
        z += __shfl_xor_sync(0xffffffffu, z, 4);
        z += __shfl_xor_sync(0xffffffffu, z, 8);
        z += __shfl_xor_sync(0xffffffffu, z, 16);
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
      // ---- V tile: O^T += V^T P^T, 8 m-tiles (16 d) x 4 k-steps (16 keys)
      if (!acquire(vit)) {
        ok = false;
        break;
      }
      const uint32_t vb = smem_u32(sm.slot[vit % NSI][0]);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t b0 = movmatrix_t(pack_bf16x2(sc[kk][0], sc[kk][1]));
        const uint32_t b1 = movmatrix_t(pack_bf16x2(sc[kk][2], sc[kk][3]));
        const int key = 16 * kk + rr + 8 * (mi >> 1);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          uint32_t a[4];
          ldsm_x4_t(a, swz(vb + (mt >> 2) * BOX, key, 2 * (mt & 3) + (mi & 1)));
          mma_bf16_16816(acc[mt], a, b0, b1);
        }
      }
      __syncwarp();
      fence_proxy_async_shared();
      if (lane == 0) mbar_arrive(&sm.empty[vit % NSI]);
    }

    // ---- epilogue: thread holds d = 16 mt + gq (acc[mt][0/1]) and 16 mt + gq + 8
    // (acc[mt][2/3]) of its rows 2c4, 2c4+1 (position my_pos, heads my_h, my_h + 1);
    // the 8 lanes of a quad column write 16 consecutive bytes per store
    if (ok && my_valid) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float inv = 1.f / den[r];
        __nv_bfloat16* o = out + (((long long)b * s.Hq + g * G + my_h + r) * s.N + my_pos) * D;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          o[16 * mt + gq] = __float2bfloat16_rn(acc[mt][r] * inv);
          o[16 * mt + gq + 8] = __float2bfloat16_rn(acc[mt][2 + r] * inv);
        }
      }
    }
  }
}

constexpr size_t kSmemBytes = sizeof(SmemR) + 1024;

}  // namespace

cudaError_t launch_attn_prefill_tc(const Shape& s, const void* q, const void* k, const void* v, const int32_t* idx,
                                   const float* s_sel, void* out, cudaStream_t st, const DevCtx& ctx) {
  if (s.d != D || s.S != S || s.G != G || s.K > KMAX || s.C > MAXC || s.nw > 32) return cudaErrorNotSupported;
  CUtensorMap tmk, tmv;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)s.N, (uint64_t)s.B * s.Hkv};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)s.N * D * 2};
  const uint32_t box[3] = {64, (uint32_t)S, 1};
  cudaError_t e = make_tmap_bf16(&tmk, k, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tmv, v, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = ensure_dynamic_smem((const void*)attn_ring_kernel, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((s.N + BP - 1) / BP, s.Hkv, s.B);
  attn_ring_kernel<<<grid, THREADS, kSmemBytes, st>>>(s, tmk, tmv, (const __nv_bfloat16*)q, idx, s_sel,
                                                      (__nv_bfloat16*)out, ctx);
  return cudaGetLastError();
}

}  // namespace hils
