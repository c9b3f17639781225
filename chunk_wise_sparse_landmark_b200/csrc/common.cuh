// Device-side building blocks shared by the HiLS kernels (sm_100a).
//
// Everything here is hand-written PTX or plain CUDA: bounded mbarrier waits
// (each wait gives up after a clock64 budget, records a timeout in the
// per-device status word and lets the kernel return), 1-D bulk copies and
// tiled tensor copies (TMA), warp-level bf16 MMA and ldmatrix, and small
// numeric helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define HILS_DI __device__ __forceinline__

namespace hils {

// ---------------------------------------------------------------- status ---
// Bits of the per-device status word (read and cleared by hils_sync_status).
enum : unsigned { kStatusTimeout = 1u, kStatusBadIndex = 2u };

struct DevCtx {
  unsigned* status;       // per-device status word
  long long wait_budget;  // clock64 cycles per bounded wait
  int inject;             // test hook: 1 = producers issue no copies, so the waits run out
};

HILS_DI void raise_status(const DevCtx& ctx, unsigned bit) { atomicOr(ctx.status, bit); }

// ---------------------------------------------------------------- types ----
HILS_DI float to_f32(float x) { return x; }
HILS_DI float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> HILS_DI T from_f32(float x);
template <> HILS_DI float from_f32<float>(float x) { return x; }
template <> HILS_DI __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// two bf16 packed in a 32-bit word -> two floats (exact widening)
HILS_DI float2 bf16x2_to_f32x2(uint32_t w) {
  float2 r;
  r.x = __uint_as_float(w << 16);
  r.y = __uint_as_float(w & 0xffff0000u);
  return r;
}
HILS_DI uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// order-preserving map float -> uint32 (larger float -> larger key)
HILS_DI uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

HILS_DI uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

// -------------------------------------------------------------- mbarrier ---
HILS_DI void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
HILS_DI void fence_barrier_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
HILS_DI void fence_proxy_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

HILS_DI void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)) : "memory");
}
HILS_DI void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// try_wait without a suspend-time hint: the hardware's own bounded wait, after
// which the caller re-polls (measured: parking waiting threads with a hint made
// the ring-fed kernels a few percent slower).
HILS_DI bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on phase `parity`.  Returns false (and records a timeout) if the
// phase did not complete within the budget; the caller must then stop issuing
// work that depends on the barrier and let the kernel finish.
HILS_DI bool mbar_wait(uint64_t* bar, uint32_t parity, const DevCtx& ctx) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > ctx.wait_budget) {
      raise_status(ctx, kStatusTimeout);
      return false;
    }
  }
  return true;
}

// ------------------------------------------------------------------ TMA ----
// 1-D bulk copy global -> shared, completion counted on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
HILS_DI void tma_load_1d(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Tiled tensor copies (tensor map in param/const/global memory).
HILS_DI void tma_load_2d(void* dst_smem, const void* tmap, int32_t x, int32_t y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst_smem)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
HILS_DI void tma_load_3d(void* dst_smem, const void* tmap, int32_t x, int32_t y, int32_t z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst_smem)),
      "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
HILS_DI void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// --------------------------------------------------------- warp-level MMA ---
// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
HILS_DI void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
HILS_DI void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
HILS_DI void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// -------------------------------------------------- tcgen05 / tensor memory ---
// Allocation is warp-wide; the TMEM address (lane << 16 | column) is written
// to shared memory.
HILS_DI void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
HILS_DI void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
HILS_DI void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
HILS_DI void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
HILS_DI void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// arrive on `bar` once every tcgen05 operation issued so far by this thread has completed
HILS_DI void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 in, fp32 accumulate)
HILS_DI void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::
          "r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T
HILS_DI void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::
          "r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, both K-major.
HILS_DI constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Shared-memory matrix descriptor for a K-major operand stored as 128-byte
// rows with the 128-byte swizzle (8-row atoms of 1024 B, atoms 1024 B apart).
// `addr` may be advanced by 32 B per 16-element K step inside an atom.
HILS_DI uint64_t sdesc_k_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                  // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;        // stride byte offset: 8-row atoms
  d |= (uint64_t)1u << 46;                  // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                  // 128-byte swizzle
  return d;
}
// 32 lanes x 32 consecutive 32-bit columns -> 32 registers per thread
HILS_DI void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
HILS_DI void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns <- 16 registers per thread
HILS_DI void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle:
// 64 MN-elements per 128-byte row, rows of consecutive K 128 B apart in
// 8-row (1024 B) atoms; `lbo` = bytes between 64-element MN blocks, `sbo` =
// bytes between 8-row K groups.
HILS_DI uint64_t sdesc_mn_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;  // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;  // 128-byte swizzle
  return d;
}

HILS_DI void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
HILS_DI void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------ reductions ---
HILS_DI float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
HILS_DI float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// ------------------------------------------------------ chunk-list form ---
// A selection list (one idx row) holds strictly ascending candidate chunks of
// its position, c in [0, ncand), followed by -1 padding; hils_score_topk
// writes exactly this form.  An entry is accepted iff it is a candidate and
// lies above every earlier entry, a negative entry counting as +inf (so that
// nothing after the first -1 is accepted).  Every attention kernel applies
// this one rule, and reports (kStatusBadIndex) any entry other than -1 that
// it drops, so that the passes agree on what they attend.
//
// Warp form: lane j holds entries j (a) and j + 32 (b); entries at or past K
// are absent.  Returns the two entries with every rejected one replaced by -1
// and sets `bad` (warp-uniform) if a non-padding entry was dropped.
HILS_DI void accept_list_warp(int& a, int& b, int K, int ncand, bool& bad) {
  const int lane = threadIdx.x & 31;
  const bool pa = lane < K, pb = lane + 32 < K;
  const int ka = (!pa || a < 0) ? 0x7fffffff : a;
  const int kb = (!pb || b < 0) ? 0x7fffffff : b;
  // exclusive prefix max of the keys over the list order a_0..a_31, b_0..b_31
  int ia = ka, ib = kb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int xa = __shfl_up_sync(0xffffffffu, ia, o), xb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia = max(ia, xa);
      ib = max(ib, xb);
    }
  }
  const int tot_a = __shfl_sync(0xffffffffu, ia, 31);
  int pa_ex = __shfl_up_sync(0xffffffffu, ia, 1), pb_ex = __shfl_up_sync(0xffffffffu, ib, 1);
  if (lane == 0) {
    pa_ex = -1;
    pb_ex = tot_a;
  } else {
    pb_ex = max(pb_ex, tot_a);
  }
  const bool oka = pa && a >= 0 && a < ncand && a > pa_ex;
  const bool okb = pb && b >= 0 && b < ncand && b > pb_ex;
  const bool bada = pa && a != -1 && !oka, badb = pb && b != -1 && !okb;
  bad = __any_sync(0xffffffffu, bada || badb);
  a = oka ? a : -1;
  b = okb ? b : -1;
}

// The same rule for entry x of a list in memory (sequential; K <= 64).
HILS_DI bool list_entry_accepted(const int32_t* list, int x, int ncand) {
  int prev = -1;
  for (int y = 0; y < x; ++y) {
    const int c = list[y];
    prev = c < 0 ? 0x7fffffff : max(prev, c);
  }
  const int c = list[x];
  return c >= 0 && c < ncand && c > prev;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace hils
