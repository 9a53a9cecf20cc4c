// api.cu -- the extern "C" entry points of libsparda: argument validation on
// the host, workspace sizing, and dispatch to the kernels.  Nothing here
// synchronizes the device; every launch is checked with cudaGetLastError.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/sparda.h"
#include "common.cuh"
#include "internal.h"

using namespace sparda;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// shapes every entry point shares; returns a status
int sparda::check_params(const sparda_params *p) {
  if (!p) return SPARDA_EINVAL;
  if (p->B < 0 || p->Hq <= 0 || p->G <= 0 || p->T < 1 || p->k < 0 || p->n_init < 0 ||
      p->n_local < 0)
    return SPARDA_EINVAL;
  if (p->Hq % p->G != 0) return SPARDA_EINVAL;
  if (p->d != kD || p->blk != kBlk) return SPARDA_EUNSUPPORTED;
  const int r = p->Hq / p->G;
  if (r != 1 && r != 2 && r != 4 && r != 8 && r != 16) return SPARDA_EUNSUPPORTED;
  if (p->k > 1024 || p->n_init > 64 || p->n_local > 64) return SPARDA_EUNSUPPORTED;
  if (p->k + p->n_init + p->n_local < 1) return SPARDA_EINVAL;
  if (p->tune) {
    const sparda_tuning &t = *p->tune;
    if (t.select_chunk < 0 || t.attn_ctas < 0 || t.prefetch_ctas < 0 || t.attn_wait_cycles < 0)
      return SPARDA_EINVAL;
    if (t.attn_stages != 0 && t.attn_stages != 2 && t.attn_stages != 3 && t.attn_stages != 4 &&
        t.attn_stages != 6)
      return SPARDA_EINVAL;
    if (t.attn_split_kv > 0 && t.attn_stages > 3) return SPARDA_EINVAL;  // 2 or 3 stages only
  }
  return SPARDA_OK;
}

namespace {

int from_cuda(cudaError_t e) { return e == cudaSuccess ? SPARDA_OK : SPARDA_ECUDA; }

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// calls that do not read per-sequence lengths refuse them rather than
// silently using T for every sequence

bool stride_ok(long long s) { return s > 0 && (s % 8) == 0; }

}  // namespace

namespace sparda {
// fetched through the runtime, so the library keeps no link-time dependency
// on libcuda
void *current_context() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  CUcontext c = nullptr;
  return fn(&c) == CUDA_SUCCESS ? static_cast<void *>(c) : nullptr;
}
}  // namespace sparda

// shared by the block-grid and window-grid entry points
namespace {
int head_softmax_select(const sparda_params *p, const void *Q, int nf, int q_start, float tau,
                        const void *kc, int32_t *idx, void *ws, size_t ws_bytes,
                        int32_t *dev_status, sparda_stream_t stream, int pool) {
  if (nf < 1 || q_start < 0 || q_start >= p->T) return SPARDA_EINVAL;
  if (!(tau == tau) || tau > 3.0e38f) return SPARDA_EINVAL;  // NaN or infinite
  if (nf > 16) return SPARDA_EUNSUPPORTED;
  if (p->B == 0) return SPARDA_OK;
  if (!Q || !kc || !idx) return SPARDA_EINVAL;
  if (!aligned16(Q) || !aligned16(kc) || !aligned16(idx)) return SPARDA_EINVAL;
  const HsmPlan pl = plan_head_softmax(*p, nf, pool);
  if (!head_softmax_supported(pl, nf)) return SPARDA_EUNSUPPORTED;
  if (pl.ws_bytes > 0 && (!ws || ws_bytes < pl.ws_bytes || !aligned16(ws))) return SPARDA_EWORKSPACE;
  const float t = tau > 0.f ? tau : sqrtf((float)p->d);
  return from_cuda(launch_head_softmax(*p, pl, static_cast<const uint16_t *>(Q), nf, q_start, t,
                                       static_cast<const uint16_t *>(kc), idx, ws, dev_status,
                                       reinterpret_cast<cudaStream_t>(stream), pool));
}
}  // namespace

extern "C" {

int sparda_version(void) { return 100; }

const char *sparda_status_string(int status) {
  switch (status) {
    case SPARDA_OK: return "SPARDA_OK";
    case SPARDA_EINVAL: return "SPARDA_EINVAL: invalid argument (null/misaligned pointer or bad shape)";
    case SPARDA_EUNSUPPORTED: return "SPARDA_EUNSUPPORTED: shape outside this version (d=128, blk=64, Hq/G in {1,2,4,8,16})";
    case SPARDA_ECUDA: return "SPARDA_ECUDA: a CUDA call or kernel launch failed";
    case SPARDA_ERANGE: return "SPARDA_ERANGE: a block id outside the sequence was skipped on the device";
    case SPARDA_ETIMEOUT: return "SPARDA_ETIMEOUT: a bounded device-side wait gave up";
    case SPARDA_EWORKSPACE: return "SPARDA_EWORKSPACE: workspace missing or too small";
    default: return "SPARDA: unknown status";
  }
}

int sparda_status_from_device(int32_t word) {
  if (word & SPARDA_DEV_LAYOUT) return SPARDA_ECUDA;
  if (word & SPARDA_DEV_TIMEOUT) return SPARDA_ETIMEOUT;
  if (word & SPARDA_DEV_RANGE) return SPARDA_ERANGE;
  return SPARDA_OK;
}

size_t sparda_workspace_size(int op, const sparda_params *p, int nq, int nf) {
  if (check_params(p) != SPARDA_OK) return 0;
  switch (op) {
    case SPARDA_OP_SELECT:
      return nq < 1 ? 0 : plan_select(*p, nq, nf < 1 ? 1 : nf).ws_bytes;
    case SPARDA_OP_SELECT_WINDOWS:
      return nq < 1 ? 0 : plan_select(*p, nq, nf < 1 ? 1 : nf, 4).ws_bytes;
    case SPARDA_OP_HEAD_SOFTMAX:
      return nq != 1 || nf < 1 ? 0 : plan_head_softmax(*p, nf, 1).ws_bytes;
    case SPARDA_OP_HEAD_SOFTMAX_WINDOWS:
      return nq != 1 || nf < 1 ? 0 : plan_head_softmax(*p, nf, 4).ws_bytes;
    case SPARDA_OP_ATTN_DECODE:
      return plan_decode(*p).ws_bytes;
    case SPARDA_OP_ATTN_PREFILL:
      return nq < 1 ? 0 : prefill_ws_bytes(*p, nq);
    default:
      return 0;
  }
}

int sparda_compress_keys(const sparda_params *p, const void *K, long long bg_stride,
                         long long tok_stride, float *kc_f32, void *kc_bf16,
                         sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (p->B == 0) return SPARDA_OK;
  if (!K || (!kc_f32 && !kc_bf16)) return SPARDA_EINVAL;
  if (!aligned16(K) || (kc_f32 && !aligned16(kc_f32)) || (kc_bf16 && !aligned16(kc_bf16)))
    return SPARDA_EINVAL;
  if (!stride_ok(tok_stride) || !stride_ok(bg_stride) || tok_stride < kD) return SPARDA_EINVAL;
  if (p->G > 1 && bg_stride < (long long)p->T * tok_stride) return SPARDA_EINVAL;
  return from_cuda(launch_compress(*p, static_cast<const uint16_t *>(K), bg_stride, tok_stride,
                                   kc_f32, static_cast<uint16_t *>(kc_bf16),
                                   reinterpret_cast<cudaStream_t>(stream)));
}

int sparda_append_kv(const sparda_params *p, int pos, const void *K_new, const void *V_new,
                     void *K, void *V, long long bg_stride, long long blk_stride, float *kc_f32,
                     void *kc_bf16, sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (!p->seq_len && (pos < 0 || pos >= p->T)) return SPARDA_EINVAL;
  if (p->B == 0) return SPARDA_OK;
  if (!K_new || !V_new || !K || !V || (!kc_f32 && !kc_bf16)) return SPARDA_EINVAL;
  if (!aligned16(K_new) || !aligned16(V_new) || !aligned16(K) || !aligned16(V) ||
      (kc_f32 && !aligned16(kc_f32)) || (kc_bf16 && !aligned16(kc_bf16)))
    return SPARDA_EINVAL;
  if (!stride_ok(bg_stride) || !stride_ok(blk_stride) || blk_stride < (long long)kBlk * kD)
    return SPARDA_EINVAL;
  return from_cuda(launch_append(*p, pos, static_cast<const uint16_t *>(K_new),
                                 static_cast<const uint16_t *>(V_new), static_cast<uint16_t *>(K),
                                 static_cast<uint16_t *>(V), bg_stride, blk_stride, kc_f32,
                                 static_cast<uint16_t *>(kc_bf16),
                                 reinterpret_cast<cudaStream_t>(stream)));
}

int sparda_append_windows(const sparda_params *p, int pos, const void *K, long long bg_stride,
                          long long blk_stride, int win, int stride, float *kw_f32, void *kw_bf16,
                          sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (win != 32 || stride != 16) return SPARDA_EUNSUPPORTED;
  if (!p->seq_len && (pos < 0 || pos >= p->T)) return SPARDA_EINVAL;
  if (p->B == 0) return SPARDA_OK;
  if (!K || (!kw_f32 && !kw_bf16)) return SPARDA_EINVAL;
  if (!aligned16(K) || (kw_f32 && !aligned16(kw_f32)) || (kw_bf16 && !aligned16(kw_bf16)))
    return SPARDA_EINVAL;
  if (!stride_ok(bg_stride) || !stride_ok(blk_stride) || blk_stride < (long long)kBlk * kD)
    return SPARDA_EINVAL;
  return from_cuda(launch_append_windows(*p, pos, static_cast<const uint16_t *>(K), bg_stride,
                                         blk_stride, kw_f32, static_cast<uint16_t *>(kw_bf16),
                                         reinterpret_cast<cudaStream_t>(stream)));
}

int sparda_compress_windows(const sparda_params *p, const void *K, long long bg_stride,
                            long long tok_stride, int win, int stride, float *kw_f32,
                            void *kw_bf16, sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (win != 32 || stride != 16) return SPARDA_EUNSUPPORTED;
  if (p->B == 0) return SPARDA_OK;
  if (!K || (!kw_f32 && !kw_bf16)) return SPARDA_EINVAL;
  if (!aligned16(K) || (kw_f32 && !aligned16(kw_f32)) || (kw_bf16 && !aligned16(kw_bf16)))
    return SPARDA_EINVAL;
  if (!stride_ok(tok_stride) || !stride_ok(bg_stride) || tok_stride < kD) return SPARDA_EINVAL;
  if (p->G > 1 && bg_stride < (long long)p->T * tok_stride) return SPARDA_EINVAL;
  return from_cuda(launch_compress_runs(*p, static_cast<const uint16_t *>(K), bg_stride,
                                        tok_stride, win, stride, kw_f32,
                                        static_cast<uint16_t *>(kw_bf16),
                                        reinterpret_cast<cudaStream_t>(stream)));
}

int sparda_forecast_select_windows(const sparda_params *p, const void *F, int nq, int nf,
                                   int q_start, const void *kw, int win, int stride,
                                   int32_t *idx, void *ws, size_t ws_bytes, int32_t *dev_status,
                                   sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (win != 32 || stride != 16) return SPARDA_EUNSUPPORTED;
  if (nq < 1 || nf < 1 || q_start < 0 || (long long)q_start + nq > p->T) return SPARDA_EINVAL;
  if (nf > 16) return SPARDA_EUNSUPPORTED;
  if (p->B == 0) return SPARDA_OK;
  if (!F || !kw || !idx) return SPARDA_EINVAL;
  if (!aligned16(F) || !aligned16(kw) || !aligned16(idx)) return SPARDA_EINVAL;
  const SelectPlan pl = plan_select(*p, nq, nf, 4);
  if (!select_supported(pl)) return SPARDA_EUNSUPPORTED;
  if (pl.ws_bytes > 0 && (!ws || ws_bytes < pl.ws_bytes || !aligned16(ws))) return SPARDA_EWORKSPACE;
  return from_cuda(launch_select(*p, pl, static_cast<const uint16_t *>(F), nq, nf, q_start,
                                 static_cast<const uint16_t *>(kw), idx, ws, dev_status,
                                 reinterpret_cast<cudaStream_t>(stream), 4));
}

int sparda_head_softmax_select(const sparda_params *p, const void *Q, int nf, int q_start,
                               float tau, const void *kc, int32_t *idx, void *ws,
                               size_t ws_bytes, int32_t *dev_status, sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  return head_softmax_select(p, Q, nf, q_start, tau, kc, idx, ws, ws_bytes, dev_status, stream,
                             1);
}

int sparda_head_softmax_select_windows(const sparda_params *p, const void *Q, int nf,
                                       int q_start, float tau, const void *kw, int win,
                                       int stride, int32_t *idx, void *ws, size_t ws_bytes,
                                       int32_t *dev_status, sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (win != 32 || stride != 16) return SPARDA_EUNSUPPORTED;
  return head_softmax_select(p, Q, nf, q_start, tau, kw, idx, ws, ws_bytes, dev_status, stream,
                             4);
}

int sparda_forecast_select(const sparda_params *p, const void *F, int nq, int nf, int q_start,
                           const void *kc, int32_t *idx, void *ws, size_t ws_bytes,
                           int32_t *dev_status, sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (nq < 1 || nf < 1 || q_start < 0 || (long long)q_start + nq > p->T) return SPARDA_EINVAL;
  if (nf > 16) return SPARDA_EUNSUPPORTED;
  if (p->B == 0) return SPARDA_OK;
  if (!F || !kc || !idx) return SPARDA_EINVAL;
  if (!aligned16(F) || !aligned16(kc) || !aligned16(idx)) return SPARDA_EINVAL;
  const SelectPlan pl = plan_select(*p, nq, nf);
  if (!select_supported(pl)) return SPARDA_EUNSUPPORTED;
  if (pl.ws_bytes > 0 && (!ws || ws_bytes < pl.ws_bytes || !aligned16(ws))) return SPARDA_EWORKSPACE;
  return from_cuda(launch_select(*p, pl, static_cast<const uint16_t *>(F), nq, nf, q_start,
                                 static_cast<const uint16_t *>(kc), idx, ws, dev_status,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

int sparda_prefetch_blocks(const sparda_params *p, const void *host_kv, const int32_t *idx,
                           void *slots, int skip_resident, int n_ctas, int32_t *dev_status,
                           sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (n_ctas < 0) return SPARDA_EINVAL;
  if (p->B == 0) return SPARDA_OK;
  if (!host_kv || !idx || !slots) return SPARDA_EINVAL;
  if (!aligned16(host_kv) || !aligned16(idx) || !aligned16(slots)) return SPARDA_EINVAL;
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, host_kv) != cudaSuccess) {
    (void)cudaGetLastError();
    return SPARDA_EINVAL;
  }
  if (attr.type != cudaMemoryTypeHost || attr.devicePointer == nullptr) return SPARDA_EINVAL;
  const uint16_t *dev_view = static_cast<const uint16_t *>(attr.devicePointer);
  if (!aligned16(dev_view)) return SPARDA_EINVAL;
  return from_cuda(launch_prefetch(*p, dev_view, idx, static_cast<uint16_t *>(slots),
                                   skip_resident, n_ctas, dev_status,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

int sparda_sparse_attn_decode(const sparda_params *p, const void *Q, const void *K,
                              const void *V, long long bg_stride, long long blk_stride,
                              const int32_t *idx, int addr_mode, void *O, void *ws,
                              size_t ws_bytes, int32_t *dev_status, sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (addr_mode != SPARDA_ADDR_LOGICAL && addr_mode != SPARDA_ADDR_SLOT) return SPARDA_EINVAL;
  if (p->B == 0) return SPARDA_OK;
  if (!Q || !K || !V || !idx || !O) return SPARDA_EINVAL;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(idx) || !aligned16(O))
    return SPARDA_EINVAL;
  if (!stride_ok(bg_stride) || !stride_ok(blk_stride) || blk_stride < (long long)kBlk * kD)
    return SPARDA_EINVAL;
  const DecodePlan pl = plan_decode(*p);
  if (pl.ws_bytes > 0 && (!ws || ws_bytes < pl.ws_bytes || !aligned16(ws))) return SPARDA_EWORKSPACE;
  return from_cuda(launch_attn_decode(*p, pl, static_cast<const uint16_t *>(Q),
                                      static_cast<const uint16_t *>(K),
                                      static_cast<const uint16_t *>(V), bg_stride, blk_stride,
                                      idx, addr_mode, static_cast<uint16_t *>(O), ws, dev_status,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

// ---- device slot cache ----------------------------------------------------
static int cache_args_ok(const sparda_params *p, int C) {
  const int S = p->k + p->n_init + p->n_local;
  return C >= S && C >= 1 && C <= kMaxCacheSlots;
}

// device view of a page-locked, mapped host buffer (null if it is not one)
static const uint16_t *mapped_device_view(const void *host) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, host) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (attr.type != cudaMemoryTypeHost || attr.devicePointer == nullptr) return nullptr;
  const uint16_t *v = static_cast<const uint16_t *>(attr.devicePointer);
  return aligned16(v) ? v : nullptr;
}

int sparda_cache_plan(const sparda_params *p, int C, const int32_t *idx, int32_t *block_of,
                      int32_t *hand, int32_t *phys, int32_t *fetch, int32_t *dev_status,
                      sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (!cache_args_ok(p, C)) return SPARDA_EINVAL;
  if (p->B == 0) return SPARDA_OK;
  if (!idx || !block_of || !hand || !phys || !fetch) return SPARDA_EINVAL;
  return from_cuda(launch_cache_plan(*p, C, idx, block_of, hand, phys, fetch, dev_status,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

int sparda_prefetch_cached(const sparda_params *p, int C, const void *host_kv,
                           const int32_t *idx, const int32_t *phys, const int32_t *fetch,
                           void *cache, int n_ctas, int32_t *dev_status, sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (!cache_args_ok(p, C) || n_ctas < 0) return SPARDA_EINVAL;
  if (p->B == 0) return SPARDA_OK;
  if (!host_kv || !idx || !phys || !fetch || !cache) return SPARDA_EINVAL;
  if (!aligned16(host_kv) || !aligned16(cache)) return SPARDA_EINVAL;
  const uint16_t *dev_view = mapped_device_view(host_kv);
  if (!dev_view) return SPARDA_EINVAL;
  return from_cuda(launch_prefetch_cached(*p, C, dev_view, idx, phys, fetch,
                                          static_cast<uint16_t *>(cache), n_ctas, dev_status,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int sparda_forecast_select_cached(const sparda_params *p, const void *F, int nf, int q_start,
                                  const void *kc, int32_t *idx, void *ws, size_t ws_bytes, int C,
                                  int32_t *block_of, int32_t *hand, int32_t *phys, int32_t *fetch,
                                  const void *host_kv, void *cache, int32_t *dev_status,
                                  sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (nf < 1 || q_start < 0 || q_start >= p->T) return SPARDA_EINVAL;
  if (nf > 16) return SPARDA_EUNSUPPORTED;
  if (!cache_args_ok(p, C)) return SPARDA_EINVAL;
  if (p->B == 0) return SPARDA_OK;
  if (!F || !kc || !idx || !block_of || !hand || !phys || !fetch || !host_kv || !cache)
    return SPARDA_EINVAL;
  if (!aligned16(F) || !aligned16(kc) || !aligned16(idx) || !aligned16(host_kv) ||
      !aligned16(cache))
    return SPARDA_EINVAL;
  const uint16_t *dev_view = mapped_device_view(host_kv);
  if (!dev_view) return SPARDA_EINVAL;
  const SelectPlan pl = plan_select(*p, 1, nf);
  if (!select_supported(pl) || pl.tensor_scores) return SPARDA_EUNSUPPORTED;
  if (pl.ws_bytes > 0 && (!ws || ws_bytes < pl.ws_bytes || !aligned16(ws))) return SPARDA_EWORKSPACE;
  SelCache cc;
  cc.C = C;
  cc.block_of = block_of;
  cc.hand = hand;
  cc.phys = phys;
  cc.fetch = fetch;
  cc.cache = static_cast<uint16_t *>(cache);
  cc.host_kv = dev_view;
  return from_cuda(launch_select(*p, pl, static_cast<const uint16_t *>(F), 1, nf, q_start,
                                 static_cast<const uint16_t *>(kc), idx, ws, dev_status,
                                 reinterpret_cast<cudaStream_t>(stream), 1, &cc));
}

int sparda_sparse_attn_decode_cached(const sparda_params *p, int C, const void *Q,
                                     const void *cache, const int32_t *idx, const int32_t *phys,
                                     void *O, void *ws, size_t ws_bytes, int32_t *dev_status,
                                     sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (!cache_args_ok(p, C)) return SPARDA_EINVAL;
  if (p->B == 0) return SPARDA_OK;
  if (!Q || !cache || !idx || !phys || !O) return SPARDA_EINVAL;
  if (!aligned16(Q) || !aligned16(cache) || !aligned16(idx) || !aligned16(phys) || !aligned16(O))
    return SPARDA_EINVAL;
  const DecodePlan pl = plan_decode(*p);
  if (pl.ws_bytes > 0 && (!ws || ws_bytes < pl.ws_bytes || !aligned16(ws))) return SPARDA_EWORKSPACE;
  const long long blk_elems = 2LL * kBlk * kD;  // K block then V block
  const uint16_t *K = static_cast<const uint16_t *>(cache);
  return from_cuda(launch_attn_decode(*p, pl, static_cast<const uint16_t *>(Q), K,
                                      K + (long long)kBlk * kD, (long long)C * blk_elems,
                                      blk_elems, idx, SPARDA_ADDR_PHYS,
                                      static_cast<uint16_t *>(O), ws, dev_status,
                                      reinterpret_cast<cudaStream_t>(stream), phys, C));
}

int sparda_sparse_attn_prefill(const sparda_params *p, const void *Q, int nq, int q_start,
                               const void *K, const void *V, long long bg_stride,
                               long long tok_stride, const int32_t *idx, void *O, void *ws,
                               size_t ws_bytes, int32_t *dev_status, sparda_stream_t stream) {
  int st = check_params(p);
  if (st != SPARDA_OK) return st;
  if (nq < 1 || q_start < 0 || (long long)q_start + nq > p->T) return SPARDA_EINVAL;
  if (p->B == 0) return SPARDA_OK;
  if (!Q || !K || !V || !idx || !O) return SPARDA_EINVAL;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(idx) || !aligned16(O))
    return SPARDA_EINVAL;
  if (!stride_ok(bg_stride) || !stride_ok(tok_stride) || tok_stride < kD) return SPARDA_EINVAL;
  if (tok_stride != kD) return SPARDA_EUNSUPPORTED;  // rows of a block must be contiguous
  const size_t need = prefill_ws_bytes(*p, nq);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return SPARDA_EWORKSPACE;
  return from_cuda(launch_attn_prefill(*p, static_cast<const uint16_t *>(Q), nq, q_start,
                                       static_cast<const uint16_t *>(K),
                                       static_cast<const uint16_t *>(V), bg_stride, tok_stride,
                                       idx, static_cast<uint16_t *>(O), ws, ws_bytes, dev_status,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
