// internal.h -- launchers shared between the kernels and the C-ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/sparda.h"

namespace sparda {

// Launch a kernel that may start before the previous kernel on the stream
// has finished (programmatic stream serialization); the kernel itself waits
// for that kernel (pdl_wait) before it touches global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// The three parts of a query's block set (eq. B_l(i) of the pages):
// initial [0, init_hi), candidates [cand_lo, cand_hi), local [local_lo, c].
struct BlockParts {
  int c, init_hi, cand_lo, cand_hi, local_lo;
};

__host__ __device__ inline BlockParts block_parts(int pos, int blk, int n_init, int n_local) {
  BlockParts r;
  r.c = pos / blk;
  r.local_lo = r.c - n_local + 1;
  if (r.local_lo < 0) r.local_lo = 0;
  r.init_hi = n_init < r.local_lo ? n_init : r.local_lo;
  r.cand_lo = n_init;
  r.cand_hi = r.local_lo > r.cand_lo ? r.local_lo : r.cand_lo;
  return r;
}

// ---- compress -------------------------------------------------------------
cudaError_t launch_compress(const sparda_params &p, const uint16_t *K, long long bg_stride,
                            long long tok_stride, float *kc32, uint16_t *kc16,
                            cudaStream_t stream);

// mean of every run of `rows` positions starting at multiples of `step`
// (blocks: 64/64, the window grid: 32/16)
cudaError_t launch_compress_runs(const sparda_params &p, const uint16_t *K, long long bg_stride,
                                 long long tok_stride, int rows, int step, float *kc32,
                                 uint16_t *kc16, cudaStream_t stream);

// one decode token on the window grid: the key of the window it completes
cudaError_t launch_append_windows(const sparda_params &p, int pos, const uint16_t *K,
                                  long long bg_stride, long long blk_stride, float *kw32,
                                  uint16_t *kw16, cudaStream_t stream);

// one decode token: write its K/V rows at `pos`, recompute its block's key
cudaError_t launch_append(const sparda_params &p, int pos, const uint16_t *K_new,
                          const uint16_t *V_new, uint16_t *K, uint16_t *V, long long bg_stride,
                          long long blk_stride, float *kc32, uint16_t *kc16, cudaStream_t stream);

// ---- select ---------------------------------------------------------------
struct SelectPlan {
  long long n_problems;  // B * nq * G
  int ncand_max;         // candidates of a query at the end of the sequence
  int CH;                // candidate blocks scored per thread block
  int n_chunks;          // thread blocks per problem
  int kc;                // candidates kept per chunk: min(k, CH)
  int tensor_scores;     // 1: chunk of query tokens scored by the tcgen05 product
  size_t ws_bytes;
};
// The slot cache of the cached decode selection (C == 0: none): per (b, g)
// C slots of one layer, their blocks and clock hand, the step's slot map and
// fetch flags, and the device view of the mapped host K|V blocks.
struct SelCache {
  int C;
  int32_t *block_of;        // [B][G][C]
  int32_t *hand;            // [B][G]
  int32_t *phys;            // [B][G][S]
  int32_t *fetch;           // [B][G][S]
  uint16_t *cache;          // [B][G][C][2][blk][d]
  const uint16_t *host_kv;  // [B][G][NB][2][blk][d]
};
// pool = 1: one compressed key per block; pool = 4: the window grid (32-token
// windows at stride 16), a block scoring as the best window inside it
SelectPlan plan_select(const sparda_params &p, int nq, int nf, int pool = 1);
// windows of 32 tokens at stride 16 that fit in T tokens
__host__ __device__ inline int window_count(int T) { return T >= 32 ? (T - 32) / 16 + 1 : 0; }
// prefill (select_prefill.cu): scores of a token chunk on the tensor cores,
// then one warp per (token, group) row ranks them
constexpr int kPrefillTensorMinQ = 64;  // query tokens from which the product pays
size_t prefill_select_ws_bytes(const sparda_params &p, int nq, int pool = 1);
cudaError_t launch_select_prefill(const sparda_params &p, const uint16_t *F, int nq, int q_start,
                                  const uint16_t *kc, int32_t *idx, void *ws, int32_t *status,
                                  cudaStream_t stream, int pool = 1);
int select_supported(const SelectPlan &plan);
cudaError_t launch_select(const sparda_params &p, const SelectPlan &plan, const uint16_t *F,
                          int nq, int nf, int q_start, const uint16_t *kc, int32_t *idx,
                          void *ws, int32_t *status, cudaStream_t stream, int pool = 1,
                          const SelCache *cache = nullptr);

// the original selector's per-head softmax form (decode: one query token);
// pool as plan_select
struct HsmPlan {
  long long n_problems;  // B * G
  int ncand_max;         // candidates of a query at the end of the sequence
  int CH;                // seen blocks per thread block
  int n_chunks;          // thread blocks per problem
  int rows_cap;          // head-score slots per (problem, head) in the workspace
  size_t ws_bytes;
};
HsmPlan plan_head_softmax(const sparda_params &p, int nf, int pool);
int head_softmax_supported(const HsmPlan &plan, int nf);
cudaError_t launch_head_softmax(const sparda_params &p, const HsmPlan &plan, const uint16_t *Q,
                                int nf, int q_start, float tau, const uint16_t *kc, int32_t *idx,
                                void *ws, int32_t *status, cudaStream_t stream, int pool);

// ---- prefetch -------------------------------------------------------------
cudaError_t launch_prefetch(const sparda_params &p, const uint16_t *host_kv_dev,
                            const int32_t *idx, uint16_t *slots, int skip_resident, int n_ctas,
                            int32_t *dev_status, cudaStream_t stream);

// ---- decode attention -----------------------------------------------------
struct DecodePlan {
  int S;            // list entries per (query, group) pair
  long long n_cta;      // most thread blocks a launch may use (sizes the workspace)
  long long n_cta_min;  // fewest thread blocks the per-CTA list capacity allows
  int max_cover;    // most thread blocks any pair's entries can span
  // workspace layout, 256-byte aligned regions: segment outputs at 0, their
  // (max, sum) at ws_ml_off, one ticket word per pair at ws_ticket_off
  size_t ws_ml_off, ws_ticket_off, ws_ticket_bytes;
  size_t ws_bytes;  // total
};
DecodePlan plan_decode(const sparda_params &p);
DecodePlan plan_gather(const sparda_params &p, long long pairs);
// one query per (sequence, token, group) "pair", each with its own block list
// (addr_mode SPARDA_ADDR_PHYS: entry e reads block slot phys[e] < n_slots)
cudaError_t launch_gather_attn(const sparda_params &p, const DecodePlan &pl, int nq, int q_start,
                               const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                               long long bg_stride, long long blk_stride, const int32_t *idx,
                               int addr_mode, uint16_t *O, void *ws, int32_t *dev_status,
                               cudaStream_t stream, const int32_t *phys = nullptr,
                               int n_slots = 0);
cudaError_t launch_attn_decode(const sparda_params &p, const DecodePlan &plan,
                               const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                               long long bg_stride, long long blk_stride, const int32_t *idx,
                               int addr_mode, uint16_t *O, void *ws, int32_t *dev_status,
                               cudaStream_t stream, const int32_t *phys = nullptr,
                               int n_slots = 0);

// ---- device slot cache (cache.cu) -------------------------------------------
constexpr int kMaxCacheSlots = 4096;
cudaError_t launch_cache_plan(const sparda_params &p, int C, const int32_t *idx,
                              int32_t *block_of, int32_t *hand, int32_t *phys, int32_t *fetch,
                              int32_t *dev_status, cudaStream_t stream);
cudaError_t launch_prefetch_cached(const sparda_params &p, int C, const uint16_t *host_kv_dev,
                                   const int32_t *idx, const int32_t *phys, const int32_t *fetch,
                                   uint16_t *cache, int n_ctas, int32_t *dev_status,
                                   cudaStream_t stream);

// ---- prefill attention ----------------------------------------------------
size_t prefill_ws_bytes(const sparda_params &p, int nq);
cudaError_t launch_attn_prefill(const sparda_params &p, const uint16_t *Q, int nq, int q_start,
                                const uint16_t *K, const uint16_t *V, long long bg_stride,
                                long long tok_stride, const int32_t *idx, uint16_t *O, void *ws,
                                size_t ws_bytes, int32_t *dev_status, cudaStream_t stream);

// The CUDA context current on this thread (null if none could be had).  A
// device reset or a new primary context reloads the library's module, which
// gives kernel attributes and device symbols new values, so host-side caches
// of them are keyed on the context as well as the device.
void *current_context();

// the rules every entry point applies to its sparda_params (shapes, this
// version's limits, the tuning fields); returns a status
int check_params(const sparda_params *p);

// the caller's launch choices (sparda_params::tune), or all zero: the
// library's own
inline const sparda_tuning &tuning(const sparda_params &p) {
  static const sparda_tuning kNone = {};
  return p.tune ? *p.tune : kNone;
}

}  // namespace sparda
