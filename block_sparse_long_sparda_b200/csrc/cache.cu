// cache.cu -- a device slot cache for the selected K/V blocks across decode
// steps: find which of a step's selected blocks the (sequence, group)
// already holds in its device slots, give every other one a slot, and copy
// only those from pinned host memory.
//
// Pages cited: [p4 <section>] = the article "SparDA: a fourth projection that
// lets sparse attention prefetch its own KV cache" (ai.thesatyajit.com);
// [p1 <section>] = the SparDA summary page at deepresearch2agi.pages.dev.
//
// [p4 "The fourth projection", Algorithm 2]: layer l+1's blocks are fetched
// from CPU pinned memory on a prefetch stream while layer l computes; [p4
// "What this doesn't fix"]: that transfer is bounded by the host link.  The
// pages give no cache policy; this one is the plainest: C slots per (b, g),
// block_of[c] = the block slot c holds (-1: empty), and a clock hand.  A
// selected block that is held is a hit and keeps its slot; every other
// valid entry, in list order, takes the next slot past the hand that holds
// none of this step's blocks, and the hand moves one further.
//
// Design (B200): the plan is tiny integer work per (b, g) -- one warp each.
// The warp stages its slot map and list in shared memory, finds the hits in
// parallel (lane per entry, a broadcast scan of the map), and one lane
// places the misses in order (the policy is sequential by definition).  The
// copy is the gather of prefetch.cu (16-byte zero-copy loads from the mapped
// host buffer) over the entries marked for fetching, which each CTA first
// lists a tile at a time.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sparda {

namespace {

constexpr int kCpWarps = 4;
constexpr int kCpThreads = kCpWarps * 32;

__host__ __device__ inline int plan_words(int C, int S) { return C + 2 * S + (C + 31) / 32; }

__global__ void __launch_bounds__(kCpThreads) cache_plan_kernel(
    const int32_t *__restrict__ idx, int32_t *__restrict__ block_of, int32_t *__restrict__ hand,
    int32_t *__restrict__ phys, int32_t *__restrict__ fetch, long long pairs, int S, int C, int NB,
    int32_t *status) {
  extern __shared__ int32_t csm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long pair = (long long)blockIdx.x * kCpWarps + warp;
  if (pair >= pairs) return;  // warp-uniform; the kernel uses no block barrier
  int32_t *blk = csm + (size_t)warp * plan_words(C, S);  // [C] block held by each slot
  int32_t *ids = blk + C;                                 // [S] this step's list
  int32_t *ph = ids + S;                                  // [S] slot, or -1 / miss marker
  uint32_t *used = reinterpret_cast<uint32_t *>(ph + S);  // [C/32] slots holding this step's blocks
  const int words = (C + 31) / 32;
  for (int c = lane; c < C; c += 32) blk[c] = block_of[pair * C + c];
  for (int s = lane; s < S; s += 32) ids[s] = idx[pair * S + s];
  for (int w = lane; w < words; w += 32) used[w] = 0u;
  __syncwarp();
  // hits, in parallel: lane per entry, every lane scanning the slot map
  constexpr int kMiss = -2;
  for (int s = lane; s < S; s += 32) {
    const int j = ids[s];
    int p = -1;
    if (j >= 0 && j < NB) {
      p = kMiss;
      for (int c = 0; c < C; ++c) {
        if (blk[c] == j) {
          p = c;
          break;
        }
      }
      if (p >= 0) atomicOr(&used[p >> 5], 1u << (p & 31));
    } else if (j >= NB) {
      flag_status(status, SPARDA_DEV_RANGE);
    }
    ph[s] = p;
  }
  __syncwarp();
  // misses, in list order, by one lane: the clock hand's next slot that holds
  // none of this step's blocks (one exists: at most S - 1 slots are taken
  // while a miss is placed, and C >= S)
  if (lane == 0) {
    int h = hand[pair];
    if (h < 0 || h >= C) h = 0;
    for (int s = 0; s < S; ++s) {
      if (ph[s] != kMiss) continue;
      int guard = 0;
      while (((used[h >> 5] >> (h & 31)) & 1u) && guard < C) {
        h = (h + 1 == C) ? 0 : h + 1;
        ++guard;
      }
      if (guard >= C) {  // cannot happen when C >= S; leave the entry unplaced
        ph[s] = -1;
        flag_status(status, SPARDA_DEV_RANGE);
        continue;
      }
      blk[h] = ids[s];
      used[h >> 5] |= 1u << (h & 31);
      ph[s] = C + h;  // marked for fetching
      h = (h + 1 == C) ? 0 : h + 1;
    }
    hand[pair] = h;
  }
  __syncwarp();
  for (int c = lane; c < C; c += 32) block_of[pair * C + c] = blk[c];
  for (int s = lane; s < S; s += 32) {
    const int v = ph[s];
    phys[pair * S + s] = v >= C ? v - C : v;
    fetch[pair * S + s] = v >= C ? 1 : 0;
  }
}

constexpr int kPfThreads = 256;
constexpr int kPairBytes = 2 * kBlk * kD * 2;            // K + V block, 32 KB
constexpr int kVecPerThread = kPairBytes / 16 / kPfThreads;  // 8

// Entries are taken a tile at a time: the tile's fetch flags are read at
// once (one load latency, not one per entry) and the marked entries listed
// in shared memory, then each listed block is copied by the whole CTA.
constexpr int kPfTile = 128;

__global__ void __launch_bounds__(kPfThreads) prefetch_cached_kernel(
    const uint16_t *__restrict__ host_kv, const int32_t *__restrict__ idx,
    const int32_t *__restrict__ phys, const int32_t *__restrict__ fetch,
    uint16_t *__restrict__ cache, long long n_entries, int S, int C, int NB, int32_t *status) {
  __shared__ long long s_ent[kPfTile];
  __shared__ int s_j[kPfTile], s_c[kPfTile];
  __shared__ int s_n;
  const int tid = threadIdx.x;
  for (long long base = (long long)blockIdx.x * kPfTile; base < n_entries;
       base += (long long)gridDim.x * kPfTile) {
    if (tid == 0) s_n = 0;
    __syncthreads();
    if (tid < kPfTile) {
      const long long ent = base + tid;
      if (ent < n_entries && fetch[ent]) {
        const int j = idx[ent], c = phys[ent];
        if (j < 0 || j >= NB || c < 0 || c >= C) {
          flag_status(status, SPARDA_DEV_RANGE);
        } else {
          const int slot = atomicAdd(&s_n, 1);
          s_ent[slot] = ent;
          s_j[slot] = j;
          s_c[slot] = c;
        }
      }
    }
    __syncthreads();
    const int n = s_n;
    for (int q = 0; q < n; ++q) {
      const long long bg = s_ent[q] / S;
      const uint4 *src = reinterpret_cast<const uint4 *>(
          host_kv + (bg * NB + s_j[q]) * (long long)(kPairBytes / 2));
      uint4 *dst =
          reinterpret_cast<uint4 *>(cache + (bg * C + s_c[q]) * (long long)(kPairBytes / 2));
      uint4 v[kVecPerThread];
#pragma unroll
      for (int u = 0; u < kVecPerThread; ++u) v[u] = ldg_plain(src + u * kPfThreads + tid);
#pragma unroll
      for (int u = 0; u < kVecPerThread; ++u) stg_stream(dst + u * kPfThreads + tid, v[u]);
    }
    __syncthreads();  // the list is rebuilt for the next tile
  }
}

}  // namespace

cudaError_t launch_cache_plan(const sparda_params &p, int C, const int32_t *idx,
                              int32_t *block_of, int32_t *hand, int32_t *phys, int32_t *fetch,
                              int32_t *dev_status, cudaStream_t stream) {
  const long long pairs = (long long)p.B * p.G;
  if (pairs == 0) return cudaSuccess;
  const int S = p.k + p.n_init + p.n_local;
  const int NB = (p.T + kBlk - 1) / kBlk;
  const size_t smem = (size_t)kCpWarps * plan_words(C, S) * 4;
  static size_t raised[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem > 48 * 1024 && raised[dev] < smem) {
    const cudaError_t e = cudaFuncSetAttribute(
        cache_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    raised[dev] = smem;
  }
  cache_plan_kernel<<<(unsigned)ceil_div_ll(pairs, kCpWarps), kCpThreads, smem, stream>>>(
      idx, block_of, hand, phys, fetch, pairs, S, C, NB, dev_status);
  return cudaGetLastError();
}

cudaError_t launch_prefetch_cached(const sparda_params &p, int C, const uint16_t *host_kv_dev,
                                   const int32_t *idx, const int32_t *phys, const int32_t *fetch,
                                   uint16_t *cache, int n_ctas, int32_t *dev_status,
                                   cudaStream_t stream) {
  const int S = p.k + p.n_init + p.n_local;
  const long long n_entries = (long long)p.B * p.G * S;
  if (n_entries == 0) return cudaSuccess;
  const int NB = (p.T + kBlk - 1) / kBlk;
  if (n_ctas <= 0) {
    const int forced = tuning(p).prefetch_ctas;
    n_ctas = forced > 0 ? forced : std::min(64, 16 + 2 * p.B);
  }
  n_ctas = (int)std::min<long long>(n_ctas, ceil_div_ll(n_entries, kPfTile));
  prefetch_cached_kernel<<<n_ctas, kPfThreads, 0, stream>>>(host_kv_dev, idx, phys, fetch, cache,
                                                            n_entries, S, C, NB, dev_status);
  return cudaGetLastError();
}

}  // namespace sparda
