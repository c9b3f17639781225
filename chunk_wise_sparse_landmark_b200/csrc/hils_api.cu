// C ABI of libhils.so (declared in include/hils.h): argument validation,
// dispatch to the kernels, the per-device status word and error strings.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "hils.h"
#include "launch.h"

namespace hils {
namespace {

__device__ unsigned g_status_word;  // per device: bits of kStatus*

thread_local char g_err[512] = "";
long long g_wait_budget = 0;  // 0 = default
int g_inject = 0;
std::mutex g_mu;
unsigned* g_status_ptr[64] = {nullptr};

hils_status_t fail(hils_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

hils_status_t cuda_fail(cudaError_t e, const char* where) {
  return fail(HILS_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// Resolve the device address of this device's status word once per device.
hils_status_t dev_ctx(DevCtx* ctx) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(HILS_ERR_CUDA, "device ordinal %d out of range", dev);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_status_word);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
      g_status_ptr[dev] = (unsigned*)p;
    }
    ctx->status = g_status_ptr[dev];
  }
  // ~2 s at 2 GHz unless overridden by the test hook
  ctx->wait_budget = g_wait_budget > 0 ? g_wait_budget : 4000000000LL;
  ctx->inject = g_inject;
  return HILS_OK;
}

bool aligned16(const void* p) { return p && ((uintptr_t)p & 15u) == 0; }

// page-locked host memory (a host-resident decode cache)
bool host_resident(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

// The operations whose shape coverage is checked on the host, before any
// launch: a shape no kernel serves returns HILS_ERR_UNSUPPORTED.
enum Op {
  kOpSummaries,
  kOpScorePrefill,
  kOpScoreDecode,
  kOpAttnPrefill,
  kOpAttnDecode,
  kOpPrefillHost,
  kOpPrefillBwd,
  kOpNone
};

// Kernel coverage per operation (the dispatchers in the .cu files serve
// exactly these shapes; anything else would reach no kernel).
const char* uncovered(const Shape& s, Op op) {
  if (s.dtype == HILS_F32) {
    const bool d_ok = s.d == 32 || s.d == 64 || s.d == 128;
    const bool s_ok = s.S == 16 || s.S == 32 || s.S == 64;
    if (!d_ok) return "f32 needs d in {32, 64, 128}";
    if (!s_ok) return "f32 needs S in {16, 32, 64}";
    const bool summ = !(s.d == 32 && s.S == 64);
    const bool score = !(s.d == 128 && s.G == 8);
    const bool dec = (s.d == 64 || s.d == 128) && (s.S == 32 || s.S == 64);
    switch (op) {
      case kOpSummaries: return summ ? nullptr : "f32 summaries: no kernel for d = 32 with S = 64";
      case kOpScorePrefill: return score ? nullptr : "f32 prefill scoring: no kernel for d = 128 with G = 8";
      case kOpAttnDecode: return dec ? nullptr : "f32 decode attention needs d in {64, 128} and S in {32, 64}";
      case kOpPrefillBwd: return nullptr;
      case kOpPrefillHost:
        if (!summ) return "f32 summaries: no kernel for d = 32 with S = 64";
        return score ? nullptr : "f32 prefill scoring: no kernel for d = 128 with G = 8";
      default: return nullptr;
    }
  }
  if (s.d != 128 || s.S != 64) return "bf16 needs d = 128 and S = 64";
  switch (op) {
    case kOpScorePrefill:
    case kOpAttnPrefill:
    case kOpPrefillHost:
      if (s.G != 4) return "bf16 prefill needs G = Hq / Hkv = 4";
      if (op != kOpScorePrefill && s.C > 8192) return "bf16 prefill attention needs N / S <= 8192";
      return nullptr;
    default: return nullptr;
  }
}

hils_status_t make_shape(const hils_config_t* cfg, Shape* s, Op op) {
  if (!cfg) return fail(HILS_ERR_INVALID_ARG, "cfg is NULL");
  const hils_config_t& c = *cfg;
  if (c.batch < 1 || c.seq_len < 1 || c.n_q_heads < 1 || c.n_kv_heads < 1 || c.head_dim < 1 || c.chunk < 1 ||
      c.window < 1 || c.top_k < 1)
    return fail(HILS_ERR_INVALID_ARG, "sizes must be positive (B=%d N=%d Hq=%d Hkv=%d d=%d S=%d W=%d K=%d)",
                c.batch, c.seq_len, c.n_q_heads, c.n_kv_heads, c.head_dim, c.chunk, c.window, c.top_k);
  if (c.n_q_heads % c.n_kv_heads) return fail(HILS_ERR_INVALID_ARG, "Hq %% Hkv != 0");
  if (c.window % c.chunk || c.window < c.chunk) return fail(HILS_ERR_INVALID_ARG, "W must be a positive multiple of S");
  if (c.dtype != HILS_F32 && c.dtype != HILS_BF16) return fail(HILS_ERR_INVALID_ARG, "unknown dtype %d", c.dtype);
  if (c.query_block < 0) return fail(HILS_ERR_INVALID_ARG, "query_block < 0");
  if (!(c.scale >= 0.f) || isinf(c.scale)) return fail(HILS_ERR_INVALID_ARG, "scale must be finite and >= 0");
  s->B = c.batch;
  s->N = c.seq_len;
  s->Hq = c.n_q_heads;
  s->Hkv = c.n_kv_heads;
  s->G = c.n_q_heads / c.n_kv_heads;
  s->d = c.head_dim;
  s->S = c.chunk;
  s->W = c.window;
  s->nw = c.window / c.chunk;
  s->K = c.top_k;
  s->C = c.seq_len / c.chunk;
  s->M = c.query_block;
  s->scale = c.scale > 0.f ? c.scale : 1.0f / sqrtf((float)c.head_dim);
  s->dtype = c.dtype;
  // kernel coverage
  const bool g_ok = s->G == 1 || s->G == 2 || s->G == 4 || s->G == 8;
  if (!g_ok) return fail(HILS_ERR_UNSUPPORTED, "G = Hq/Hkv = %d not in {1,2,4,8}", s->G);
  if (s->K > 64) return fail(HILS_ERR_UNSUPPORTED, "K = %d > 64", s->K);
  if (s->nw > 32) return fail(HILS_ERR_UNSUPPORTED, "W/S = %d > 32", s->nw);
  if (const char* why = uncovered(*s, op)) return fail(HILS_ERR_UNSUPPORTED, "%s", why);
  return HILS_OK;
}

#define HILS_TRY(x)                      \
  do {                                   \
    hils_status_t _st = (x);             \
    if (_st != HILS_OK) return _st;      \
  } while (0)

#define HILS_LAUNCH(expr, where)                                                                  \
  do {                                                                                            \
    cudaError_t _e = (expr);                                                                      \
    if (_e == cudaErrorNotSupported) return fail(HILS_ERR_UNSUPPORTED, "%s: no kernel for this shape", where); \
    if (_e != cudaSuccess) return cuda_fail(_e, where);                                           \
  } while (0)

size_t esize(const Shape& s) { return s.dtype == HILS_F32 ? 4 : 2; }

// ------------------------------------------------ host-memory prefill path ---
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Offsets, in the caller's workspace, of the device copies of the inputs and of
// every intermediate tensor of hils_prefill_host.
struct HostLayout {
  size_t q, k, v, qlmk, ksum, bsum, idx, ssel, out, attn, h, wd, wu, qt, total;
};
// one (sequence, KV group) piece of a shape: its G query heads and one KV head
Shape piece_shape(const Shape& s) {
  Shape sub = s;
  sub.B = 1;
  sub.Hq = s.G;
  sub.Hkv = 1;
  return sub;
}
HostLayout host_layout(const Shape& s, int rank) {
  HostLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += up256(bytes);
    return o;
  };
  const size_t e = esize(s);
  L.q = take((size_t)s.B * s.Hq * s.N * s.d * e);
  L.k = take((size_t)s.B * s.Hkv * s.N * s.d * e);
  L.v = take((size_t)s.B * s.Hkv * s.N * s.d * e);
  L.qlmk = take((size_t)s.B * s.Hq * s.C * s.d * e);
  L.ksum = take((size_t)s.B * s.Hq * s.C * s.d * e);
  L.bsum = take((size_t)s.B * s.Hq * s.C * 4);
  L.idx = take((size_t)s.B * s.Hkv * s.N * s.K * 4);
  L.ssel = take((size_t)s.B * s.Hq * s.N * s.K * 4);
  L.out = take((size_t)s.B * s.Hq * s.N * s.d * e);
  L.attn = take(s.dtype == HILS_BF16 ? attn_prefill_tc_workspace(piece_shape(s)) : 0);
  if (rank > 0) {
    const size_t dm = (size_t)s.Hq * s.d;  // the supported Q-Cal width
    L.h = take((size_t)s.B * s.N * dm * e);
    L.wd = take((size_t)rank * dm * e);
    L.wu = take((size_t)s.Hq * s.d * rank * e);
    L.qt = take((size_t)s.B * s.Hq * s.N * s.d * e);
  }
  L.total = off;
  return L;
}

// Two copy streams (uploads, downloads) and a pool of events per device.  The
// whole enqueue sequence of one call holds g_pipe_mu, so concurrent calls never
// record an event that another call is about to wait on.
struct Pipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t* ev = nullptr;
  int nev = 0;
};
Pipe g_pipe[64];
std::mutex g_pipe_mu;

hils_status_t get_pipe(int dev, int nev, Pipe** pp) {
  Pipe& p = g_pipe[dev];
  cudaError_t e;
  if (!p.in) {
    e = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreate");
  }
  if (!p.out) {
    e = cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreate");
  }
  if (p.nev < nev) {
    cudaEvent_t* ev = new cudaEvent_t[nev];
    for (int i = 0; i < p.nev; ++i) ev[i] = p.ev[i];
    for (int i = p.nev; i < nev; ++i) {
      e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
      if (e != cudaSuccess) {
        for (int j = p.nev; j < i; ++j) cudaEventDestroy(ev[j]);
        delete[] ev;
        return cuda_fail(e, "cudaEventCreate");
      }
    }
    delete[] p.ev;
    p.ev = ev;
    p.nev = nev;
  }
  *pp = &p;
  return HILS_OK;
}

#define HILS_CK(expr, where)                                \
  do {                                                      \
    cudaError_t _e = (expr);                                \
    if (_e != cudaSuccess) return cuda_fail(_e, where);     \
  } while (0)

// one NVTX range per C-ABI call, named after the call (a no-op unless a
// profiler that records NVTX is attached)
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define HILS_NVTX NvtxRange hils_nvtx_range_(__func__)

}  // namespace
}  // namespace hils

using namespace hils;

extern "C" {

const char* hils_version(void) { return "hils-b200 1.0"; }

const char* hils_last_error(void) { return g_err; }

void hils_set_wait_budget(int64_t cycles) { g_wait_budget = cycles > 0 ? cycles : 0; }

void hils_set_fault_injection(int32_t mode) { g_inject = mode == 1 ? 1 : 0; }

hils_status_t hils_build_summaries(const hils_config_t* cfg, const void* k, const void* q_lmk, void* k_sum,
                                   float* b_sum, void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, kOpSummaries));
  if (!aligned16(k) || !aligned16(q_lmk) || !aligned16(k_sum) || !aligned16(b_sum))
    return fail(HILS_ERR_INVALID_ARG, "hils_build_summaries: NULL or unaligned pointer");
  if (s.dtype == HILS_BF16 && (((uintptr_t)k | (uintptr_t)q_lmk) & 31u))
    return fail(HILS_ERR_INVALID_ARG, "hils_build_summaries: bf16 k and q_lmk must be 32-byte aligned");
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  HILS_LAUNCH(launch_summaries(s, k, q_lmk, k_sum, b_sum, (cudaStream_t)stream, ctx), "summaries");
  return HILS_OK;
}

hils_status_t hils_build_summaries_shared(const hils_config_t* cfg, const void* k, const void* q_shared,
                                          void* k_sum, float* b_sum, void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, kOpSummaries));
  if (!aligned16(k) || !aligned16(q_shared) || !aligned16(k_sum) || !aligned16(b_sum))
    return fail(HILS_ERR_INVALID_ARG, "hils_build_summaries_shared: NULL or unaligned pointer");
  if (s.dtype == HILS_BF16 && (((uintptr_t)k | (uintptr_t)q_shared) & 31u))
    return fail(HILS_ERR_INVALID_ARG, "hils_build_summaries_shared: bf16 k and q_shared must be 32-byte aligned");
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  HILS_LAUNCH(launch_summaries(s, k, q_shared, k_sum, b_sum, (cudaStream_t)stream, ctx, true), "summaries_shared");
  return HILS_OK;
}

size_t hils_workspace_bytes(const hils_config_t* cfg, int32_t which, int32_t qcal_rank) {
  Shape s;
  const Op op = which == HILS_WS_SCORE_PREFILL ? kOpScorePrefill
                : which == HILS_WS_SCORE_DECODE ? kOpScoreDecode
                : which == HILS_WS_ATTN_DECODE  ? kOpAttnDecode
                : which == HILS_WS_PREFILL_HOST ? kOpPrefillHost
                : which == HILS_WS_ATTN_PREFILL ? kOpAttnPrefill
                : which == HILS_WS_PREFILL_BWD  ? kOpPrefillBwd
                                                : kOpNone;
  if (op == kOpNone) {
    fail(HILS_ERR_INVALID_ARG, "unknown workspace kind %d", which);
    return (size_t)-1;
  }
  if (make_shape(cfg, &s, op) != HILS_OK) return (size_t)-1;
  switch (which) {
    case HILS_WS_SCORE_PREFILL: {
      size_t b = 0;
      if (s.dtype == HILS_BF16) b += score_tc_workspace(s);
      if (qcal_rank > 0) b += (size_t)s.B * s.Hq * s.N * s.d * esize(s);  // q~
      return b;
    }
    case HILS_WS_SCORE_DECODE:
      return decode_score_workspace(s);
    case HILS_WS_ATTN_DECODE:
      return decode_attn_workspace(s);
    case HILS_WS_PREFILL_HOST:
      return host_layout(s, qcal_rank > 0 ? qcal_rank : 0).total;
    case HILS_WS_ATTN_PREFILL:
      return s.dtype == HILS_BF16 ? attn_prefill_tc_workspace(s) : 0;
    case HILS_WS_PREFILL_BWD:
      return prefill_bwd_workspace(s);
  }
  return (size_t)-1;
}

hils_status_t hils_score_topk(const hils_config_t* cfg, const void* q, const hils_qcal_t* qcal, const void* k_sum,
                              const float* b_sum, int32_t* idx, float* s_sel, void* workspace, size_t ws_bytes,
                              int32_t decode, void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, decode ? kOpScoreDecode : kOpScorePrefill));
  if (decode != 0 && decode != 1) return fail(HILS_ERR_INVALID_ARG, "decode must be 0 or 1");
  if (!aligned16(q) || !aligned16(k_sum) || !aligned16(b_sum) || !aligned16(idx) || !aligned16(s_sel))
    return fail(HILS_ERR_INVALID_ARG, "hils_score_topk: NULL or unaligned pointer");
  const size_t need = hils_workspace_bytes(cfg, decode ? HILS_WS_SCORE_DECODE : HILS_WS_SCORE_PREFILL,
                                           qcal ? qcal->rank : 0);
  if (need > 0 && (ws_bytes < need || !aligned16(workspace)))
    return fail(HILS_ERR_INVALID_ARG, "hils_score_topk: workspace needs %zu bytes (got %zu)", need, ws_bytes);
  if (qcal) {
    if (decode) return fail(HILS_ERR_UNSUPPORTED, "Q-Cal is a prefill-only option");
    if (!aligned16(qcal->h) || !aligned16(qcal->w_down) || !aligned16(qcal->w_up))
      return fail(HILS_ERR_INVALID_ARG, "Q-Cal: NULL or unaligned pointer");
    if (qcal->rank != 64 || qcal->d_model < 64 || qcal->d_model % 64)
      return fail(HILS_ERR_UNSUPPORTED, "Q-Cal: rank %d / d_model %d not supported", qcal->rank, qcal->d_model);
    if (s.dtype != HILS_BF16) return fail(HILS_ERR_UNSUPPORTED, "Q-Cal needs bf16");
  }
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  cudaStream_t st = (cudaStream_t)stream;
  if (decode) {
    HILS_LAUNCH(launch_score_topk_decode(s, q, k_sum, b_sum, idx, s_sel, workspace, st, ctx), "score_topk_decode");
    return HILS_OK;
  }
  const void* q_score = q;
  unsigned char* ws = (unsigned char*)workspace;
  if (qcal) {
    void* q_tilde = ws;
    ws += (size_t)s.B * s.Hq * s.N * s.d * esize(s);
    HILS_LAUNCH(launch_qcal_tc(s, q, qcal->h, qcal->w_down, qcal->w_up, qcal->rank, qcal->d_model, q_tilde, st, ctx),
                "qcal");
    q_score = q_tilde;
  }
  if (s.dtype == HILS_F32) {
    HILS_LAUNCH(launch_score_topk_simt(s, q_score, k_sum, b_sum, idx, s_sel, st, ctx), "score_topk_simt");
  } else {
    HILS_LAUNCH(launch_score_topk_tc(s, q_score, k_sum, b_sum, idx, s_sel, st, ctx), "score_topk_tc");
  }
  return HILS_OK;
}

hils_status_t hils_attn_prefill(const hils_config_t* cfg, const void* q, const void* k, const void* v,
                                const int32_t* idx, const float* s_sel, void* out, void* workspace,
                                size_t ws_bytes, void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, kOpAttnPrefill));
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(s_sel) || !aligned16(out))
    return fail(HILS_ERR_INVALID_ARG, "hils_attn_prefill: NULL or unaligned pointer");
  const bool bf16 = s.dtype == HILS_BF16;
  const bool chunked = bf16 && (workspace || ws_bytes > 0);
  if (bf16 && (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v) & 31u))
    return fail(HILS_ERR_INVALID_ARG, "hils_attn_prefill: bf16 q, k, v must be 32-byte aligned");
  if (chunked) {
    const size_t need = attn_prefill_tc_workspace(s);
    if (ws_bytes < need || !aligned16(workspace))
      return fail(HILS_ERR_INVALID_ARG, "hils_attn_prefill: workspace needs %zu bytes (got %zu)", need, ws_bytes);
  }
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  cudaStream_t st = (cudaStream_t)stream;
  if (!bf16) {
    HILS_LAUNCH(launch_attn_prefill_simt(s, q, k, v, idx, s_sel, out, st, ctx), "attn_prefill_simt");
  } else if (chunked) {
    HILS_LAUNCH(launch_attn_prefill_chunked(s, q, k, v, idx, s_sel, out, workspace, st, ctx), "attn_prefill_chunked");
  } else {
    HILS_LAUNCH(launch_attn_prefill_tc(s, q, k, v, idx, s_sel, out, st, ctx), "attn_prefill_tc");
  }
  return HILS_OK;
}

hils_status_t hils_prefill_bwd(const hils_config_t* cfg, const void* q, const void* k, const void* v,
                               const void* q_lmk, const int32_t* idx, const float* s_sel, const void* k_sum,
                               const void* dout, float* dq, float* dk, float* dv, float* dq_lmk, float* ds_sel,
                               void* workspace, size_t ws_bytes, void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, kOpPrefillBwd));
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_lmk) || !aligned16(idx) || !aligned16(s_sel) ||
      !aligned16(k_sum) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      !aligned16(dq_lmk) || (ds_sel && !aligned16(ds_sel)))
    return fail(HILS_ERR_INVALID_ARG, "hils_prefill_bwd: NULL or unaligned pointer");
  const size_t need = prefill_bwd_workspace(s);
  if (ws_bytes < need || !aligned16(workspace))
    return fail(HILS_ERR_INVALID_ARG, "hils_prefill_bwd: workspace needs %zu bytes (got %zu)", need, ws_bytes);
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  HILS_LAUNCH(launch_prefill_bwd(s, q, k, v, q_lmk, idx, s_sel, k_sum, dout, dq, dk, dv, dq_lmk, ds_sel, workspace,
                                 (cudaStream_t)stream, ctx),
              "prefill_bwd");
  return HILS_OK;
}

hils_status_t hils_prefill_host(const hils_config_t* cfg, const void* h_q, const void* h_k, const void* h_v,
                                const void* h_q_lmk, const hils_qcal_t* qcal, void* h_out, void* workspace,
                                size_t ws_bytes, void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, kOpPrefillHost));
  if (!h_q || !h_k || !h_v || !h_q_lmk || !h_out) return fail(HILS_ERR_INVALID_ARG, "hils_prefill_host: NULL host pointer");
  const int rank = qcal ? qcal->rank : 0;
  if (qcal) {
    if (!qcal->h || !qcal->w_down || !qcal->w_up) return fail(HILS_ERR_INVALID_ARG, "Q-Cal: NULL host pointer");
    if (s.dtype != HILS_BF16) return fail(HILS_ERR_UNSUPPORTED, "Q-Cal needs bf16");
    if (qcal->rank != 64 || qcal->d_model != s.Hq * s.d)
      return fail(HILS_ERR_UNSUPPORTED, "hils_prefill_host: Q-Cal rank %d / d_model %d not supported (d_model must be Hq*d)",
                  qcal->rank, qcal->d_model);
  }
  const size_t need = hils_workspace_bytes(cfg, HILS_WS_PREFILL_HOST, rank);
  if (ws_bytes < need || !aligned16(workspace))
    return fail(HILS_ERR_INVALID_ARG, "hils_prefill_host: workspace needs %zu bytes (got %zu)", need, ws_bytes);
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  int dev = 0;
  HILS_CK(cudaGetDevice(&dev), "cudaGetDevice");
  const HostLayout L = host_layout(s, rank);
  unsigned char* W = (unsigned char*)workspace;
  unsigned char *dq = W + L.q, *dk = W + L.k, *dv = W + L.v, *dql = W + L.qlmk, *dks = W + L.ksum, *dout = W + L.out;
  float* dbs = (float*)(W + L.bsum);
  int32_t* didx = (int32_t*)(W + L.idx);
  float* dss = (float*)(W + L.ssel);
  const unsigned char *hq = (const unsigned char*)h_q, *hk = (const unsigned char*)h_k, *hv = (const unsigned char*)h_v,
                      *hql = (const unsigned char*)h_q_lmk;
  unsigned char* hout = (unsigned char*)h_out;
  const size_t e = esize(s);
  const int P = s.B * s.Hkv;  // pieces: (sequence, KV group)
  const size_t nq = (size_t)s.G * s.N * s.d * e, nkv = (size_t)s.N * s.d * e, nql = (size_t)s.G * s.C * s.d * e;
  const Shape sub = piece_shape(s);  // one piece: one sequence, one KV group and its G query heads
  unsigned char* dattn = W + L.attn;
  auto piece = [&](int p, size_t* oq, size_t* okv, size_t* oql, size_t* obs, size_t* oidx, size_t* oss) {
    const size_t b = p / s.Hkv, g = p % s.Hkv, h0 = b * s.Hq + g * s.G, kv = b * s.Hkv + g;
    *oq = h0 * s.N * s.d * e;
    *okv = kv * s.N * s.d * e;
    *oql = h0 * s.C * s.d * e;
    *obs = h0 * s.C;
    *oidx = kv * s.N * s.K;
    *oss = h0 * s.N * s.K;
  };
  std::lock_guard<std::mutex> lk(g_pipe_mu);
  Pipe* pp = nullptr;
  HILS_TRY(get_pipe(dev, 2 * P + 3, &pp));
  cudaStream_t st = (cudaStream_t)stream, ci = pp->in, co = pp->out;
  cudaEvent_t ev_start = pp->ev[0], ev_all = pp->ev[1], ev_done = pp->ev[2];
  cudaEvent_t* ev_in = pp->ev + 3;
  cudaEvent_t* ev_att = pp->ev + 3 + P;
  // the copy streams start after the work already on `stream` (which may still use the workspace)
  HILS_CK(cudaEventRecord(ev_start, st), "cudaEventRecord");
  HILS_CK(cudaStreamWaitEvent(ci, ev_start, 0), "cudaStreamWaitEvent");
  HILS_CK(cudaStreamWaitEvent(co, ev_start, 0), "cudaStreamWaitEvent");
  if (!qcal) {
    for (int p = 0; p < P; ++p) {
      size_t oq, okv, oql, obs, oidx, oss;
      piece(p, &oq, &okv, &oql, &obs, &oidx, &oss);
      HILS_CK(cudaMemcpyAsync(dk + okv, hk + okv, nkv, cudaMemcpyHostToDevice, ci), "upload k");
      HILS_CK(cudaMemcpyAsync(dql + oql, hql + oql, nql, cudaMemcpyHostToDevice, ci), "upload q_lmk");
      HILS_CK(cudaMemcpyAsync(dq + oq, hq + oq, nq, cudaMemcpyHostToDevice, ci), "upload q");
      HILS_CK(cudaMemcpyAsync(dv + okv, hv + okv, nkv, cudaMemcpyHostToDevice, ci), "upload v");
      HILS_CK(cudaEventRecord(ev_in[p], ci), "cudaEventRecord");
    }
    for (int p = 0; p < P; ++p) {
      size_t oq, okv, oql, obs, oidx, oss;
      piece(p, &oq, &okv, &oql, &obs, &oidx, &oss);
      HILS_CK(cudaStreamWaitEvent(st, ev_in[p], 0), "cudaStreamWaitEvent");
      HILS_LAUNCH(launch_summaries(sub, dk + okv, dql + oql, dks + oql, dbs + obs, st, ctx), "summaries");
      if (s.dtype == HILS_F32) {
        HILS_LAUNCH(launch_score_topk_simt(sub, dq + oq, dks + oql, dbs + obs, didx + oidx, dss + oss, st, ctx),
                    "score_topk_simt");
        HILS_LAUNCH(launch_attn_prefill_simt(sub, dq + oq, dk + okv, dv + okv, didx + oidx, dss + oss, dout + oq, st, ctx),
                    "attn_prefill_simt");
      } else {
        HILS_LAUNCH(launch_score_topk_tc(sub, dq + oq, dks + oql, dbs + obs, didx + oidx, dss + oss, st, ctx),
                    "score_topk_tc");
        HILS_LAUNCH(launch_attn_prefill_chunked(sub, dq + oq, dk + okv, dv + okv, didx + oidx, dss + oss, dout + oq,
                                                dattn, st, ctx),
                    "attn_prefill_chunked");
      }
      HILS_CK(cudaEventRecord(ev_att[p], st), "cudaEventRecord");
      HILS_CK(cudaStreamWaitEvent(co, ev_att[p], 0), "cudaStreamWaitEvent");
      HILS_CK(cudaMemcpyAsync(hout + oq, dout + oq, nq, cudaMemcpyDeviceToHost, co), "download out");
    }
  } else {
    // Q-Cal: the low-rank term t = W_down h is shared by all heads, so the
    // scoring runs on the whole problem once every input is on the device
    const size_t all_q = (size_t)s.B * s.Hq * s.N * s.d * e, all_kv = (size_t)s.B * s.Hkv * s.N * s.d * e;
    const size_t all_ql = (size_t)s.B * s.Hq * s.C * s.d * e, dm = (size_t)s.Hq * s.d;
    HILS_CK(cudaMemcpyAsync(dk, hk, all_kv, cudaMemcpyHostToDevice, ci), "upload k");
    HILS_CK(cudaMemcpyAsync(dql, hql, all_ql, cudaMemcpyHostToDevice, ci), "upload q_lmk");
    HILS_CK(cudaMemcpyAsync(W + L.h, qcal->h, (size_t)s.B * s.N * dm * e, cudaMemcpyHostToDevice, ci), "upload h");
    HILS_CK(cudaMemcpyAsync(W + L.wd, qcal->w_down, (size_t)rank * dm * e, cudaMemcpyHostToDevice, ci), "upload W_down");
    HILS_CK(cudaMemcpyAsync(W + L.wu, qcal->w_up, (size_t)s.Hq * s.d * rank * e, cudaMemcpyHostToDevice, ci),
            "upload W_up");
    HILS_CK(cudaMemcpyAsync(dq, hq, all_q, cudaMemcpyHostToDevice, ci), "upload q");
    HILS_CK(cudaEventRecord(ev_all, ci), "cudaEventRecord");
    HILS_CK(cudaMemcpyAsync(dv, hv, all_kv, cudaMemcpyHostToDevice, ci), "upload v");
    HILS_CK(cudaEventRecord(ev_in[0], ci), "cudaEventRecord");
    HILS_CK(cudaStreamWaitEvent(st, ev_all, 0), "cudaStreamWaitEvent");
    HILS_LAUNCH(launch_summaries(s, dk, dql, dks, dbs, st, ctx), "summaries");
    HILS_LAUNCH(launch_qcal_tc(s, dq, W + L.h, W + L.wd, W + L.wu, rank, (int)dm, W + L.qt, st, ctx), "qcal");
    HILS_LAUNCH(launch_score_topk_tc(s, W + L.qt, dks, dbs, didx, dss, st, ctx), "score_topk_tc");
    HILS_CK(cudaStreamWaitEvent(st, ev_in[0], 0), "cudaStreamWaitEvent");
    for (int p = 0; p < P; ++p) {
      size_t oq, okv, oql, obs, oidx, oss;
      piece(p, &oq, &okv, &oql, &obs, &oidx, &oss);
      HILS_LAUNCH(launch_attn_prefill_chunked(sub, dq + oq, dk + okv, dv + okv, didx + oidx, dss + oss, dout + oq,
                                              dattn, st, ctx),
                  "attn_prefill_chunked");
      HILS_CK(cudaEventRecord(ev_att[p], st), "cudaEventRecord");
      HILS_CK(cudaStreamWaitEvent(co, ev_att[p], 0), "cudaStreamWaitEvent");
      HILS_CK(cudaMemcpyAsync(hout + oq, dout + oq, nq, cudaMemcpyDeviceToHost, co), "download out");
    }
  }
  // `stream` passes the call once the last download has landed
  HILS_CK(cudaEventRecord(ev_done, co), "cudaEventRecord");
  HILS_CK(cudaStreamWaitEvent(st, ev_done, 0), "cudaStreamWaitEvent");
  return HILS_OK;
}

hils_status_t hils_attn_decode(const hils_config_t* cfg, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* idx, const float* s_sel, void* out, void* workspace, size_t ws_bytes,
                               void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, kOpAttnDecode));
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(idx) || !aligned16(s_sel) ||
      !aligned16(out))
    return fail(HILS_ERR_INVALID_ARG, "hils_attn_decode: NULL or unaligned pointer");
  const size_t need = decode_attn_workspace(s);
  if (ws_bytes < need || !aligned16(workspace))
    return fail(HILS_ERR_INVALID_ARG, "hils_attn_decode: workspace needs %zu bytes (got %zu)", need, ws_bytes);
  if (s.dtype == HILS_F32 && (host_resident(k_cache) || host_resident(v_cache)))
    return fail(HILS_ERR_UNSUPPORTED, "hils_attn_decode: a host-resident cache needs bf16 (the fp32 kernel copies "
                                      "tiles with the bulk-copy engine)");
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  HILS_LAUNCH(launch_attn_decode(s, q, k_cache, v_cache, idx, s_sel, out, workspace, (cudaStream_t)stream, ctx),
              "attn_decode");
  return HILS_OK;
}

hils_status_t hils_attn_decode_noalloc(const hils_config_t* cfg, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* idx, const float* s_sel, void* out,
                                       void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, kOpAttnDecode));
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(idx) || !aligned16(s_sel) ||
      !aligned16(out))
    return fail(HILS_ERR_INVALID_ARG, "hils_attn_decode_noalloc: NULL or unaligned pointer");
  const size_t need = decode_attn_workspace(s), have = decode_static_scratch_bytes();
  if (need > have)
    return fail(HILS_ERR_UNSUPPORTED,
                "hils_attn_decode_noalloc: this configuration needs %zu bytes of scratch, the library's fixed "
                "scratch holds %zu; use hils_attn_decode with a workspace",
                need, have);
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  HILS_LAUNCH(launch_attn_decode_static(s, q, k_cache, v_cache, idx, s_sel, out, (cudaStream_t)stream, ctx),
              "attn_decode_noalloc");
  return HILS_OK;
}

// host checks of a paged-cache description; its device arrays are checked by
// the kernels (lengths in [1, N], pages inside the pool)
static hils_status_t paged_view(const Shape& s, const hils_paged_t* pg, DecView* dv) {
  if (!pg) return fail(HILS_ERR_INVALID_ARG, "paged cache description is NULL");
  if (!pg->seq_lens || ((uintptr_t)pg->seq_lens & 3u) || !pg->block_table || ((uintptr_t)pg->block_table & 3u))
    return fail(HILS_ERR_INVALID_ARG, "paged cache: NULL or unaligned seq_lens / block_table");
  const int need = (s.N + s.S - 1) / s.S;
  if (pg->max_pages < need)
    return fail(HILS_ERR_INVALID_ARG, "paged cache: max_pages %d < ceil(seq_len / S) = %d", pg->max_pages, need);
  if (pg->num_pages < 1) return fail(HILS_ERR_INVALID_ARG, "paged cache: num_pages %d < 1", pg->num_pages);
  dv->seq_lens = pg->seq_lens;
  dv->pages = pg->block_table;
  dv->max_pages = pg->max_pages;
  dv->num_pages = pg->num_pages;
  return HILS_OK;
}

hils_status_t hils_decode_append(const hils_config_t* cfg, const hils_paged_t* paged, const void* k_new,
                                 const void* v_new, const void* q_lmk_new, void* k_pool, void* v_pool, void* k_sum,
                                 float* b_sum, void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, kOpSummaries));
  DecView dv;
  HILS_TRY(paged_view(s, paged, &dv));
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(q_lmk_new) || !aligned16(k_pool) || !aligned16(v_pool) ||
      !aligned16(k_sum) || !aligned16(b_sum))
    return fail(HILS_ERR_INVALID_ARG, "hils_decode_append: NULL or unaligned pointer");
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  cudaStream_t st = (cudaStream_t)stream;
  HILS_LAUNCH(launch_decode_append(s, k_new, v_new, k_pool, v_pool, dv, st, ctx), "decode_append");
  HILS_LAUNCH(launch_summaries_paged(s, k_pool, q_lmk_new, k_sum, b_sum, dv, true, st, ctx), "summaries_paged");
  return HILS_OK;
}

hils_status_t hils_build_summaries_paged(const hils_config_t* cfg, const hils_paged_t* paged, const void* k_pool,
                                         const void* q_lmk, void* k_sum, float* b_sum, void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, kOpSummaries));
  DecView dv;
  HILS_TRY(paged_view(s, paged, &dv));
  if (!aligned16(k_pool) || !aligned16(q_lmk) || !aligned16(k_sum) || !aligned16(b_sum))
    return fail(HILS_ERR_INVALID_ARG, "hils_build_summaries_paged: NULL or unaligned pointer");
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  HILS_LAUNCH(launch_summaries_paged(s, k_pool, q_lmk, k_sum, b_sum, dv, false, (cudaStream_t)stream, ctx),
              "summaries_paged");
  return HILS_OK;
}

hils_status_t hils_score_topk_paged(const hils_config_t* cfg, const void* q, const hils_paged_t* paged,
                                    const void* k_sum, const float* b_sum, int32_t* idx, float* s_sel,
                                    void* workspace, size_t ws_bytes, void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, kOpScoreDecode));
  DecView dv;
  HILS_TRY(paged_view(s, paged, &dv));
  if (!aligned16(q) || !aligned16(k_sum) || !aligned16(b_sum) || !aligned16(idx) || !aligned16(s_sel))
    return fail(HILS_ERR_INVALID_ARG, "hils_score_topk_paged: NULL or unaligned pointer");
  const size_t need = decode_score_workspace(s);
  if (ws_bytes < need || !aligned16(workspace))
    return fail(HILS_ERR_INVALID_ARG, "hils_score_topk_paged: workspace needs %zu bytes (got %zu)", need, ws_bytes);
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  HILS_LAUNCH(launch_score_topk_decode(s, q, k_sum, b_sum, idx, s_sel, workspace, (cudaStream_t)stream, ctx, dv),
              "score_topk_paged");
  return HILS_OK;
}

hils_status_t hils_attn_decode_paged(const hils_config_t* cfg, const void* q, const void* k_pool, const void* v_pool,
                                     const hils_paged_t* paged, const int32_t* idx, const float* s_sel, void* out,
                                     void* workspace, size_t ws_bytes, void* stream) {
  HILS_NVTX;
  Shape s;
  HILS_TRY(make_shape(cfg, &s, kOpAttnDecode));
  DecView dv;
  HILS_TRY(paged_view(s, paged, &dv));
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(idx) || !aligned16(s_sel) ||
      !aligned16(out))
    return fail(HILS_ERR_INVALID_ARG, "hils_attn_decode_paged: NULL or unaligned pointer");
  const size_t need = decode_attn_workspace(s);
  if (ws_bytes < need || !aligned16(workspace))
    return fail(HILS_ERR_INVALID_ARG, "hils_attn_decode_paged: workspace needs %zu bytes (got %zu)", need, ws_bytes);
  if (s.dtype == HILS_F32 && (host_resident(k_pool) || host_resident(v_pool)))
    return fail(HILS_ERR_UNSUPPORTED, "hils_attn_decode_paged: a host-resident pool needs bf16");
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  HILS_LAUNCH(launch_attn_decode(s, q, k_pool, v_pool, idx, s_sel, out, workspace, (cudaStream_t)stream, ctx, dv),
              "attn_decode_paged");
  return HILS_OK;
}

hils_status_t hils_host_device_pointer(const void* host, void** device_ptr) {
  HILS_NVTX;
  if (!host || !device_ptr) return fail(HILS_ERR_INVALID_ARG, "hils_host_device_pointer: NULL argument");
  void* p = nullptr;
  const cudaError_t e = cudaHostGetDevicePointer(&p, const_cast<void*>(host), 0);
  if (e != cudaSuccess) {
    cudaGetLastError();  // clear the error state so that later calls do not report it
    return fail(HILS_ERR_INVALID_ARG, "hils_host_device_pointer: not page-locked mapped host memory (%s)",
                cudaGetErrorString(e));
  }
  *device_ptr = p;
  return HILS_OK;
}

hils_status_t hils_sync_status(void* stream) {
  HILS_NVTX;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  DevCtx ctx;
  HILS_TRY(dev_ctx(&ctx));
  unsigned word = 0;
  e = cudaMemcpy(&word, ctx.status, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  if (word) {
    const unsigned zero = 0;
    e = cudaMemcpy(ctx.status, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clear status");
  }
  if (word & kStatusTimeout) return fail(HILS_ERR_TIMEOUT, "a device wait exceeded its budget (status 0x%x)", word);
  if (word & kStatusBadIndex) return fail(HILS_ERR_INVALID_ARG, "a kernel skipped an out-of-range chunk index");
  return HILS_OK;
}

}  // extern "C"
