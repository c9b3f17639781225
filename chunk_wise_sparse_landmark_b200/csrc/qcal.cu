// Q-Cal: low-rank query calibration for chunk scoring (bf16, d = 128, rank 64).
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法
// (Method), second practical design choice: the scoring query is
// q~_i = q_i + W_up W_down h_i with rank r << d_model; it is used for the
// chunk scores only.
//
// One CTA = 128 positions of one sequence.  GEMM 1 (t = h W_down^T, 128 x 64,
// K = d_model) streams h and W_down tiles through a 3-stage TMA ring
// (128-byte swizzle) into tcgen05 MMAs with the accumulator in tensor memory.
// The epilogue warps round t to bf16 and write it into shared memory in the
// same swizzled K-major layout, where it becomes the A operand of GEMM 2
// (dq = t W_up^T, one head = 128 output columns at a time, single-buffered in
// TMEM).  For each head the epilogue adds q and stores q~ in the layout of q.
// Warp roles: 0 = TMA producer, 1 = MMA issuer / TMEM owner, 2..5 epilogue.
#include "launch.h"
#include "tmap.h"

namespace hils {
namespace {

constexpr int D = 128, R = 64, MQ = 128, KB = 64;  // KB: d_model elements per k-block
constexpr int NS = 3;
constexpr int THREADS = 192;
constexpr uint32_t A1_BYTES = MQ * 128;         // [128 rows x 64] bf16
constexpr uint32_t B1_BYTES = R * 128;          // [64 rows x 64] bf16
constexpr uint32_t B2_BYTES = D * 128;          // [128 rows x 64] bf16
constexpr uint32_t STAGE = A1_BYTES + B1_BYTES; // 24 KB (>= B2_BYTES)
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t D1COL = 0, D2COL = 128;

struct __align__(1024) SmemQ {
  unsigned char st[NS][STAGE];
  unsigned char a2[MQ * 128];  // t in bf16, K-major, 128-byte swizzle
  uint64_t full[NS], empty[NS], d1full, a2full, d2full, d2empty, done;
  uint32_t tmem;
};

__global__ void __launch_bounds__(THREADS, 1)
    qcal_kernel(Shape s, int d_model, const __grid_constant__ CUtensorMap tmh,
                const __grid_constant__ CUtensorMap tmwd, const __grid_constant__ CUtensorMap tmwu,
                const __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ q_tilde, DevCtx ctx) {
  extern __shared__ unsigned char smem_raw[];
  SmemQ& sm = *reinterpret_cast<SmemQ*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.y;
  const int i0 = blockIdx.x * MQ;
  const int NK = d_model / KB;
  const int NIT = NK + s.Hq;

  if (tid == 0) {
    for (int x = 0; x < NS; ++x) {
      mbar_init(&sm.full[x], 1);
      mbar_init(&sm.empty[x], 1);
    }
    mbar_init(&sm.d1full, 1);
    mbar_init(&sm.a2full, 4);
    mbar_init(&sm.d2full, 1);
    mbar_init(&sm.d2empty, 4);
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
    int last_round[NS] = {-1, -1, -1};
    if (lane == 0) {
      prefetch_tmap(&tmh);
      prefetch_tmap(&tmwd);
      prefetch_tmap(&tmwu);
    }
    bool ok = true;
    for (int it = 0; it < NIT && ok; ++it) {
      const int st = it % NS, rnd = it / NS;
      if (rnd > 0) ok = mbar_wait(&sm.empty[st], (rnd - 1) & 1, ctx);
      if (!ok) break;
      if (lane == 0 && ctx.inject != 1) {
        if (it < NK) {
          mbar_arrive_expect_tx(&sm.full[st], STAGE);
          tma_load_2d(sm.st[st], &tmh, it * KB, b * s.N + i0, &sm.full[st]);
          tma_load_2d(sm.st[st] + A1_BYTES, &tmwd, it * KB, 0, &sm.full[st]);
        } else {
          mbar_arrive_expect_tx(&sm.full[st], B2_BYTES);
          tma_load_2d(sm.st[st], &tmwu, 0, (it - NK) * D, &sm.full[st]);
        }
        last_round[st] = rnd;
      }
      __syncwarp();
    }
    if (lane == 0)
      for (int x = 0; x < NS; ++x)
        if (last_round[x] >= 0) mbar_wait(&sm.full[x], last_round[x] & 1, ctx);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA ------
    const uint32_t id1 = idesc_bf16_f32(MQ, R), id2 = idesc_bf16_f32(MQ, D);
    bool ok = true;
    for (int it = 0; it < NIT && ok; ++it) {
      const int st = it % NS;
      ok = mbar_wait(&sm.full[st], (it / NS) & 1, ctx);
      if (ok && it == NK) {  // GEMM 2 needs t staged by the epilogue
        ok = mbar_wait(&sm.a2full, 0, ctx);
      }
      if (ok && it > NK) ok = mbar_wait(&sm.d2empty, (it - NK - 1) & 1, ctx);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t base = smem_u32(sm.st[st]);
        if (it < NK) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ss(tmem + D1COL, sdesc_k_sw128(base + k * 32), sdesc_k_sw128(base + A1_BYTES + k * 32), id1,
                   (it > 0 || k > 0) ? 1u : 0u);
          tc_commit(&sm.empty[st]);
          if (it == NK - 1) tc_commit(&sm.d1full);
        } else {
          const uint32_t a2 = smem_u32(sm.a2);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ss(tmem + D2COL, sdesc_k_sw128(a2 + k * 32), sdesc_k_sw128(base + k * 32), id2, k > 0 ? 1u : 0u);
          tc_commit(&sm.empty[st]);
          tc_commit(&sm.d2full);
        }
      }
      __syncwarp();
    }
    if (lane == 0) {
      tc_commit(&sm.done);
      mbar_wait(&sm.done, 0, ctx);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue ----
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const int i = i0 + r;
    const bool valid = i < s.N;
    const uint32_t lane_addr = tmem + ((uint32_t)(qd * 32) << 16);
    bool ok = mbar_wait(&sm.d1full, 0, ctx);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      uint32_t t0[32], t1[32];
      tmem_ld32(lane_addr + D1COL, t0);
      tmem_ld32(lane_addr + D1COL + 32, t1);
      tmem_wait_ld();
      // t -> bf16, row r of a 128B-swizzled K-major tile
      unsigned char* row = sm.a2 + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 u;
        const uint32_t* src = c < 4 ? &t0[c * 8] : &t1[(c - 4) * 8];
        u.x = pack_bf16x2(__uint_as_float(src[0]), __uint_as_float(src[1]));
        u.y = pack_bf16x2(__uint_as_float(src[2]), __uint_as_float(src[3]));
        u.z = pack_bf16x2(__uint_as_float(src[4]), __uint_as_float(src[5]));
        u.w = pack_bf16x2(__uint_as_float(src[6]), __uint_as_float(src[7]));
        *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = u;
      }
      fence_proxy_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.a2full);
      for (int hq = 0; hq < s.Hq; ++hq) {
        ok = mbar_wait(&sm.d2full, hq & 1, ctx);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        uint32_t v[4][32];
#pragma unroll
        for (int x = 0; x < 4; ++x) tmem_ld32(lane_addr + D2COL + x * 32, v[x]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.d2empty);
        if (valid) {
          const long long off = (((long long)b * s.Hq + hq) * s.N + i) * D;
          const uint4* qs = reinterpret_cast<const uint4*>(q + off);
          uint4* qt = reinterpret_cast<uint4*>(q_tilde + off);
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const uint4 u = qs[x];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            uint32_t o[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              const float2 f = bf16x2_to_f32x2(w[y]);
              const int e = x * 8 + y * 2;
              o[y] = pack_bf16x2(f.x + __uint_as_float(v[e >> 5][e & 31]),
                                 f.y + __uint_as_float(v[(e + 1) >> 5][(e + 1) & 31]));
            }
            qt[x] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
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

cudaError_t launch_qcal_tc(const Shape& s, const void* q, const void* h, const void* w_down, const void* w_up,
                           int rank, int d_model, void* q_tilde, cudaStream_t st, const DevCtx& ctx) {
  if (s.d != D || rank != R || d_model % KB) return cudaErrorNotSupported;
  CUtensorMap tmh, tmwd, tmwu;
  {
    const uint64_t dims[2] = {(uint64_t)d_model, (uint64_t)s.B * s.N};
    const uint64_t strides[1] = {(uint64_t)d_model * 2};
    const uint32_t box[2] = {KB, MQ};
    cudaError_t e = make_tmap_bf16(&tmh, h, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
  }
  {
    const uint64_t dims[2] = {(uint64_t)d_model, (uint64_t)R};
    const uint64_t strides[1] = {(uint64_t)d_model * 2};
    const uint32_t box[2] = {KB, R};
    cudaError_t e = make_tmap_bf16(&tmwd, w_down, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
  }
  {
    const uint64_t dims[2] = {(uint64_t)R, (uint64_t)s.Hq * D};
    const uint64_t strides[1] = {(uint64_t)R * 2};
    const uint32_t box[2] = {R, D};
    cudaError_t e = make_tmap_bf16(&tmwu, w_up, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = sizeof(SmemQ) + 1024;
  cudaError_t e = ensure_dynamic_smem((const void*)qcal_kernel, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((s.N + MQ - 1) / MQ, s.B);
  qcal_kernel<<<grid, THREADS, smem, st>>>(s, d_model, tmh, tmwd, tmwu, (const __nv_bfloat16*)q,
                                           (__nv_bfloat16*)q_tilde, ctx);
  return cudaGetLastError();
}

}  // namespace hils
