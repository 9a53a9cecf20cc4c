// attn_prefill.cu -- block-sparse prefill attention: every token of a query
// chunk attends over the keys of its own block set, causal.
//
// Pages cited: [p4 <section>] = the article "SparDA: a fourth projection that
// lets sparse attention prefetch its own KV cache" (ai.thesatyajit.com);
// [p1 <section>] = the SparDA summary page at deepresearch2agi.pages.dev.
//
// [p4 "The fourth projection", Algorithm 1 / Eq. 5]: O_l = attention(Q_l,
// K_l[B_l], V_l[B_l]) with every key resident on the GPU.
//
// The chunk runs through the tcgen05 gather kernel of attn_decode.cu with one
// (token, group) pair per block list; pairs are streamed group by group so
// that the K/V the running CTAs read stays in L2.
#include "common.cuh"
#include "internal.h"

namespace sparda {

size_t prefill_ws_bytes(const sparda_params &p, int nq) {
  return plan_gather(p, (long long)p.B * nq * p.G).ws_bytes;
}

cudaError_t launch_attn_prefill(const sparda_params &p, const uint16_t *Q, int nq, int q_start,
                                const uint16_t *K, const uint16_t *V, long long bg_stride,
                                long long tok_stride, const int32_t *idx, uint16_t *O, void *ws,
                                size_t ws_bytes, int32_t *dev_status, cudaStream_t stream) {
  (void)ws_bytes;
  const DecodePlan pl = plan_gather(p, (long long)p.B * nq * p.G);
  return launch_gather_attn(p, pl, nq, q_start, Q, K, V, bg_stride, (long long)kBlk * tok_stride,
                            idx, SPARDA_ADDR_LOGICAL, O, ws, dev_status, stream);
}

}  // namespace sparda
