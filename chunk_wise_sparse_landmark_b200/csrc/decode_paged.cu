// Decode across steps on a paged, chunk-aligned KV cache.
//
// hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 实验
// (Experiments): prefill and decode latency grow sublinearly with context;
// the wmrh.cn article on HiLS: decode is 15.7x faster than full attention at
// 512K.  A decode step touches only the token's K chunks and its window, so a
// cache that grows by one token per step needs only (a) the new token's key
// and value written into place and (b) when that token completes a chunk, the
// landmark summary of that one chunk (the Method section's k'_c, b'_c, from
// the chunk's landmark query q'_c).  Rebuilding every summary each step would
// read the whole cache.
//
// The cache is a pool of one-chunk pages [num_pages, Hkv, S, d]: chunk c of
// sequence b lives in page block_table[b, c], so sequences of different
// lengths share one pool and a chunk of one KV head stays one contiguous
// S x d tile (the unit every decode kernel loads).  This file holds the append
// kernel; the summary of the completed chunk and the paged scoring and
// attention reuse the decode kernels with a page view (DecView, launch.h).
#include "launch.h"

namespace hils {
namespace {

// one CTA per sequence: element e of KV head g of the new token goes to
// position L - 1 of its page (L = seq_lens[b], the length with the new token)
template <typename E>
__global__ void decode_append_kernel(Shape s, const E* __restrict__ k_new, const E* __restrict__ v_new,
                                     E* __restrict__ k_pool, E* __restrict__ v_pool, DecView dv, DevCtx ctx) {
  const int b = blockIdx.x;
  const int L = dv_len(dv, s, b);
  if (L < 1 || L > s.N) {
    if (threadIdx.x == 0) raise_status(ctx, kStatusBadIndex);
    return;
  }
  const int pos = L - 1, c = pos / s.S, j = pos % s.S;
  for (int x = threadIdx.x; x < s.Hkv * s.d; x += blockDim.x) {
    const int g = x / s.d, e = x % s.d;
    const long long off = dv_chunk(dv, s, b, g, c);
    if (off < 0) {  // a page outside the pool: reported, never written
      if (e == 0) raise_status(ctx, kStatusBadIndex);
      continue;
    }
    const long long src = ((long long)b * s.Hkv + g) * s.d + e;
    k_pool[off + (long long)j * s.d + e] = k_new[src];
    v_pool[off + (long long)j * s.d + e] = v_new[src];
  }
}

}  // namespace

cudaError_t launch_decode_append(const Shape& s, const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                                 const DecView& dv, cudaStream_t st, const DevCtx& ctx) {
  const int threads = 256;
  if (s.dtype == 0)
    decode_append_kernel<uint32_t><<<s.B, threads, 0, st>>>(s, (const uint32_t*)k_new, (const uint32_t*)v_new,
                                                            (uint32_t*)k_pool, (uint32_t*)v_pool, dv, ctx);
  else
    decode_append_kernel<uint16_t><<<s.B, threads, 0, st>>>(s, (const uint16_t*)k_new, (const uint16_t*)v_new,
                                                            (uint16_t*)k_pool, (uint16_t*)v_pool, dv, ctx);
  return cudaGetLastError();
}

}  // namespace hils
