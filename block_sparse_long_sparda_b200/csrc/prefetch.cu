// prefetch.cu -- gather the selected K/V blocks of the next layer from pinned
// host memory into device slots, on the caller's (side) stream.
//
// Pages cited: [p4 <section>] = the article "SparDA: a fourth projection that
// lets sparse attention prefetch its own KV cache" (ai.thesatyajit.com);
// [p1 <section>] = the SparDA summary page at deepresearch2agi.pages.dev.
//
// [p4 "The fourth projection", Algorithm 2]: the blocks picked for layer l+1
// are fetched from CPU pinned memory to the GPU on a dedicated prefetch
// stream while layer l computes; [p1 "UVA异步预取管线"]: the kernel reads
// host memory directly through unified virtual addressing and its thread
// block count adapts to the batch size.
//
// Design (B200): the block ids are produced on the device by the selection
// kernel, so the copy has to be driven by the device too -- a host-driven
// copy engine transfer would need the ids back on the host (a device->host
// copy and a synchronisation per layer).  Each thread block walks (b, g, s)
// list entries with a grid stride; for a selected block it streams the 32 KB
// K|V pair over the host link with 16-byte zero-copy loads, 8 per thread in
// flight (32 KB per 256-thread block), and writes the slot with streaming
// stores.  A small, batch-dependent number of thread blocks keeps enough
// requests in flight to fill the link while leaving the SMs to the
// attention kernel running concurrently on the compute stream.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sparda {

namespace {

constexpr int kPfThreads = 256;
constexpr int kPairBytes = 2 * kBlk * kD * 2;           // K + V block, 32 KB
constexpr int kVecPerPair = kPairBytes / 16;             // 2048 x 16 B
constexpr int kVecPerThread = kVecPerPair / kPfThreads;  // 8

__global__ void __launch_bounds__(kPfThreads) prefetch_kernel(
    const uint16_t *__restrict__ host_kv, const int32_t *__restrict__ idx,
    uint16_t *__restrict__ slots, long long n_entries, int S, int NB, int cand_lo, int cand_hi,
    int skip_resident, int32_t *status, const int32_t *seq_len, int G, int T, int n_init,
    int n_local) {
  for (long long ent = blockIdx.x; ent < n_entries; ent += gridDim.x) {
    const int j = idx[ent];
    if (j < 0) continue;
    if (j >= NB) {
      if (threadIdx.x == 0) flag_status(status, SPARDA_DEV_RANGE);
      continue;
    }
    const long long bg = ent / S;
    int lo = cand_lo, hi = cand_hi;
    if (seq_len) {  // the resident initial and local blocks of this sequence
      const int len = seq_len[bg / G];
      if (len < 1 || len > T) {
        if (threadIdx.x == 0) flag_status(status, SPARDA_DEV_RANGE);
        continue;
      }
      const BlockParts bp = block_parts(len - 1, kBlk, n_init, n_local);
      lo = bp.cand_lo;
      hi = bp.cand_hi;
    }
    if (skip_resident && !(j >= lo && j < hi)) continue;
    const uint4 *src =
        reinterpret_cast<const uint4 *>(host_kv + ((bg * NB + j) * (long long)kPairBytes / 2));
    uint4 *dst = reinterpret_cast<uint4 *>(slots + ent * (long long)(kPairBytes / 2));
    uint4 v[kVecPerThread];
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) v[u] = ldg_plain(src + u * kPfThreads + threadIdx.x);
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) stg_stream(dst + u * kPfThreads + threadIdx.x, v[u]);
  }
}

}  // namespace

cudaError_t launch_prefetch(const sparda_params &p, const uint16_t *host_kv_dev,
                            const int32_t *idx, uint16_t *slots, int skip_resident, int n_ctas,
                            int32_t *dev_status, cudaStream_t stream) {
  const int S = p.k + p.n_init + p.n_local;
  const long long n_entries = (long long)p.B * p.G * S;
  if (n_entries == 0) return cudaSuccess;
  const int NB = (p.T + kBlk - 1) / kBlk;
  const BlockParts bp = block_parts(p.T - 1, kBlk, p.n_init, p.n_local);
  if (n_ctas <= 0) {
    const int forced = tuning(p).prefetch_ctas;
    // more sequences -> more concurrent host reads; bounded so the compute
    // stream keeps most SMs
    n_ctas = forced > 0 ? forced : std::min(64, 16 + 2 * p.B);
  }
  n_ctas = (int)std::min<long long>(n_ctas, n_entries);
  prefetch_kernel<<<n_ctas, kPfThreads, 0, stream>>>(host_kv_dev, idx, slots, n_entries, S, NB,
                                                     bp.cand_lo, bp.cand_hi, skip_resident,
                                                     dev_status, p.seq_len, p.G, p.T, p.n_init,
                                                     p.n_local);
  return cudaGetLastError();
}

}  // namespace sparda
