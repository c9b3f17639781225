// Warp-level building blocks for attending one 64-key x 128-dim bf16 tile
// that a warp gathers straight from global memory (L2 / HBM) into
// tensor-core fragments, with up to 8 query columns:
//
//   S^T (64 keys x 8 cols)  = K_tile (keys x d) . Q^T (d x cols)
//   O^T (128 d x 8 cols)   += V_tile^T (d x keys) . P^T (keys x cols)
//
// bf16 mma.sync m16n8k16 with fp32 accumulation.  Fragment coordinates:
// gq = lane / 4, c4 = lane % 4.
//
// * S^T: the contraction index d is permuted, consistently for K and Q: for
//   k-step ks = 4 jj + t (jj = 0,1; t = 0..3) thread c4 holds logical k
//   {2c4, 2c4+1} at physical d = 64 jj + 16 c4 + 4t + {0,1} and {2c4+8, 2c4+9}
//   at 64 jj + 16 c4 + 4t + {2,3}.  One 32-byte load therefore feeds four
//   k-steps, and the 8 key rows x 4 threads of a warp load cover whole
//   128-byte lines.  The S^T accumulator sc[mt][*] of a thread holds keys
//   16 mt + gq (elements 0, 1) and 16 mt + gq + 8 (elements 2, 3) of columns
//   2 c4 (elements 0, 2) and 2 c4 + 1 (elements 1, 3).
// * O^T: row r of m-tile mt is output dim 8 gq + mt (r = gq) or
//   64 + 8 gq + mt (r = gq + 8), so the value loads of a key row are one
//   contiguous 128-byte line per 8 threads.  acc[mt][0/1] hold dim 8 gq + mt
//   of columns 2 c4 / 2 c4 + 1; acc[mt][2/3] hold dim 64 + 8 gq + mt.
// * P^T reaches B-fragment layout by an in-register 8x8 transpose of the S^T
//   accumulator (movmatrix), after the caller has turned logits into weights.
#pragma once

#include "common.cuh"

namespace hils {

HILS_DI void ldg32(const __nv_bfloat16* p, uint32_t (&w)[8]) {
  asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
               : "l"(p));
}
HILS_DI uint4 ldg16(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// element e (0..7) of a 16-byte vector of bf16, in the low half-word
HILS_DI uint32_t half_of(const uint4& v, int e) {
  const uint32_t w = e < 2 ? v.x : e < 4 ? v.y : e < 6 ? v.z : v.w;
  return (e & 1) ? (w >> 16) : (w & 0xffffu);
}

HILS_DI uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Q^T B-fragments of column gq from that column's 128-dim row (nullptr: zero column).
HILS_DI void load_qcol(const __nv_bfloat16* row, int c4, uint32_t (&qf)[2][8]) {
#pragma unroll
  for (int jj = 0; jj < 2; ++jj) {
    if (row) {
      ldg32(row + 64 * jj + 16 * c4, qf[jj]);
    } else {
#pragma unroll
      for (int x = 0; x < 8; ++x) qf[jj][x] = 0u;
    }
  }
}

// sc (zeroed by the caller) += S^T of the tile at kc; key rows past kmax are
// read from row kmax (the caller masks them).
HILS_DI void mma_st_tile(const __nv_bfloat16* kc, int kmax, int gq, int c4, const uint32_t (&qf)[2][8],
                         float (&sc)[4][4]) {
#pragma unroll
  for (int jj = 0; jj < 2; ++jj) {
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      uint32_t ka[8], kb8[8];
      ldg32(kc + min(16 * mt + gq, kmax) * 128 + 64 * jj + 16 * c4, ka);
      ldg32(kc + min(16 * mt + gq + 8, kmax) * 128 + 64 * jj + 16 * c4, kb8);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t A[4] = {ka[2 * t], kb8[2 * t], ka[2 * t + 1], kb8[2 * t + 1]};
        mma_bf16_16816(sc[mt], A, qf[jj][2 * t], qf[jj][2 * t + 1]);
      }
    }
  }
}

// acc += O^T of the tile at vc with weights p (S^T accumulator layout, already
// final: masked entries zero).  Key rows past kmax are read from row kmax.
HILS_DI void mma_ot_tile(const __nv_bfloat16* vc, int kmax, int gq, int c4, const float (&p)[4][4],
                         float (&acc)[8][4]) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const uint32_t b0 = movmatrix_trans(pack_bf16x2(p[kk][0], p[kk][1]));
    const uint32_t b1 = movmatrix_trans(pack_bf16x2(p[kk][2], p[kk][3]));
    const int key0 = 16 * kk + 2 * c4;
    uint4 va[4][2];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = min(key0 + (e & 1) + 8 * (e >> 1), kmax);
      va[e][0] = ldg16(vc + key * 128 + 8 * gq);
      va[e][1] = ldg16(vc + key * 128 + 64 + 8 * gq);
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t A[4];
      A[0] = half_of(va[0][0], mt) | (half_of(va[1][0], mt) << 16);
      A[1] = half_of(va[0][1], mt) | (half_of(va[1][1], mt) << 16);
      A[2] = half_of(va[2][0], mt) | (half_of(va[3][0], mt) << 16);
      A[3] = half_of(va[2][1], mt) | (half_of(va[3][1], mt) << 16);
      mma_bf16_16816(acc[mt], A, b0, b1);
    }
  }
}

// reductions over the 8 threads that share a column (lanes differing in gq)
HILS_DI float col_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
}
HILS_DI float col_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  x += __shfl_xor_sync(0xffffffffu, x, 8);
  return x + __shfl_xor_sync(0xffffffffu, x, 16);
}

}  // namespace hils
