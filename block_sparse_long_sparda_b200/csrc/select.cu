// select.cu -- Forecast block selection: score every candidate block's
// compressed key with the group's Forecast vector(s), keep the k best, and
// join them with the initial and local blocks.
//
// [p4 "The fourth projection", Eq. 4]: B_{l+1} = B_init U B_local U
//   f_top(F_l Kc_{l+1}^T, k)
// [p4 "One Forecast head per GQA group"]: one Forecast vector per group, raw
//   dot products, no softmax.  With nf > 1 the kernel is the multi-head
//   baseline selector of the same section (per-head scores summed).
//
// Design (B200): the decode selection is a streaming read of Kc (256 B per
// block per group) with a tiny amount of math, so it is HBM bound.  A problem
// (one query token of one group of one sequence) is split into chunks of CH
// candidate blocks, one thread block each, so thousands of CTAs stream Kc at
// once.  Inside a CTA each half-warp scores 8 blocks per step: lane l loads
// dims [8l, 8l+8) of the 8 rows (8 x 16-byte loads in flight), multiplies by
// the Forecast slice, and a butterfly transpose-reduce (8 shuffles for 8
// rows) leaves the full score of each row in a pair of lanes.  Scores become
// orderable uint32 keys.  A chunk CTA only streams and scores, writing its
// keys to the workspace, so CTAs are short and many are in flight.  The
// chunks of a problem meet through an atomic ticket: the last CTA to finish
// (no waiting) loads every key of the problem from L2, a 4-pass 8-bit radix
// select finds the k-th key, and a block scan in block order keeps
// everything above it plus the lowest-index ties -- results come out sorted
// by block id and ties go to the lower id -- and writes init U top-k U local.
// No CTA ever waits for another.
#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"

namespace sparda {

namespace {

constexpr int kSelThreads = 256;
constexpr int kMaxCand = 32768;   // candidates one problem may have (keys fit in shared memory)
constexpr int kMaxNf = 16;

struct SelArgs {
  const uint16_t *F;
  const uint16_t *kc;
  int32_t *idx;
  uint32_t *counters;   // one ticket per problem (multi-chunk only)
  uint32_t *cand_key;   // [problem][cap] score keys (multi-chunk only)
  int nq, G, nf, NB, k, n_init, n_local, q_start, S;
  int CH, n_chunks, cap;
};

// ---------------------------------------------------------------------------
// block-wide helpers (blockDim.x == kSelThreads)
// ---------------------------------------------------------------------------

// Exclusive prefix sum over threads in thread order; `tmp` holds 33 words.
__device__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *tmp, uint32_t &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int nw = kSelThreads / 32;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t t = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += t;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < nw ? tmp[lane] : 0u;
    uint32_t incl = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane < nw) tmp[lane] = incl - w;
    if (lane == nw - 1) tmp[32] = incl;
  }
  __syncthreads();
  uint32_t r = tmp[warp] + x - v;
  total = tmp[32];
  __syncthreads();  // tmp may be reused by the next call
  return r;
}

// The k-th largest key among keys[0, n) and how many keys equal to it are
// kept.  Precondition: more than k of the keys are non-zero (valid), k >= 1.
__device__ void radix_threshold(const uint32_t *keys, int n, int k, uint32_t *hist,
                                uint32_t *bc, uint32_t &tau, int &need) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0;
  int rem = k;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    // warp-aggregated: lanes holding the same digit add once (scores cluster
    // in a few top-level bins, where plain atomics would serialise)
    for (int base = warp * 32; base < n; base += kSelThreads) {
      const int i = base + lane;
      const uint32_t u = i < n ? keys[i] : 0u;
      const bool match = i < n && (pass == 0 || ((u ^ prefix) >> (shift + 8)) == 0u);
      const uint32_t bin = match ? ((u >> shift) & 255u) : 256u;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (match && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t h[8], local = 0;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        h[b] = hist[lane * 8 + b];
        local += h[b];
      }
      uint32_t suf = local;  // inclusive suffix sum over lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t t = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += t;
      }
      uint32_t suf_next = __shfl_down_sync(0xffffffffu, suf, 1);
      if (lane == 31) suf_next = 0;
      if (suf >= (uint32_t)rem && suf_next < (uint32_t)rem) {
        uint32_t above = suf_next;
#pragma unroll
        for (int b = 7; b >= 0; --b) {
          if (above + h[b] >= (uint32_t)rem) {
            bc[0] = (uint32_t)(lane * 8 + b);
            bc[1] = (uint32_t)rem - above;
            break;
          }
          above += h[b];
        }
      }
    }
    __syncthreads();
    prefix |= bc[0] << shift;
    rem = (int)bc[1];
  }
  tau = prefix;
  need = rem;
}

// Keep keys > tau plus the first `need` keys == tau (in entry order), writing
// them in entry order.  Each thread owns E consecutive entries.  Returns the
// number kept (same value in every thread).
template <class IdOf, class Out>
__device__ int compact_kept(const uint32_t *keys, int n, int E, uint32_t tau, int need,
                            uint32_t *scan_tmp, IdOf id_of, Out out) {
  const int e0 = threadIdx.x * E;
  const int e1 = min(n, e0 + E);
  uint32_t packed = 0;
  for (int e = e0; e < e1; ++e) {
    const uint32_t u = keys[e];
    packed += (u > tau ? 0x10000u : 0u) + (u == tau ? 1u : 0u);
  }
  uint32_t total;
  const uint32_t before = block_exclusive_scan(packed, scan_tmp, total);
  uint32_t gt_b = before >> 16, eq_b = before & 0xFFFFu;
  for (int e = e0; e < e1; ++e) {
    const uint32_t u = keys[e];
    const bool gt = u > tau, eq = u == tau;
    if (gt || (eq && (int)eq_b < need)) {
      const uint32_t pos = gt_b + min(eq_b, (uint32_t)need);
      out((int)pos, u, id_of(e));
    }
    gt_b += gt;
    eq_b += eq;
  }
  return (int)((total >> 16) + min(total & 0xFFFFu, (uint32_t)need));
}

// init | top-k | local | -1 padding.  With `fill_top`, the top-k part is the
// first ntop candidates (every candidate is taken); otherwise it is written
// by the caller.
__device__ void write_set(int32_t *out, const BlockParts &bp, int ntop, int S, bool fill_top) {
  const int nloc = bp.c - bp.local_lo + 1;
  for (int s = threadIdx.x; s < S; s += kSelThreads) {
    int v;
    if (s < bp.init_hi) {
      v = s;
    } else if (s < bp.init_hi + ntop) {
      if (!fill_top) continue;
      v = bp.cand_lo + (s - bp.init_hi);
    } else if (s < bp.init_hi + ntop + nloc) {
      v = bp.local_lo + (s - bp.init_hi - ntop);
    } else {
      v = -1;
    }
    out[s] = v;
  }
}

// Butterfly transpose-reduce of 8 row partials over the 16 lanes of a
// half-warp: 3 exchange stages on lane bits 3, 2, 1 and a final pairwise sum
// leave the complete score of row (hl >> 1) in lanes hl and hl ^ 1.
__device__ __forceinline__ float transpose_reduce8x16(float (&p)[8], int hl) {
#pragma unroll
  for (int half = 4; half >= 1; half >>= 1) {
    const int lanebit = half * 2;
    const bool up = (hl & lanebit) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = up ? p[i] : p[i + half];
      const float keep = up ? p[i + half] : p[i];
      p[i] = keep + __shfl_xor_sync(0xffffffffu, send, lanebit);
    }
  }
  return p[0] + __shfl_xor_sync(0xffffffffu, p[0], 1);
}

__device__ __forceinline__ float dot8(const float *f, uint4 v) {
  float s = f[0] * bf16_lo(v.x);
  s = fmaf(f[1], bf16_hi(v.x), s);
  s = fmaf(f[2], bf16_lo(v.y), s);
  s = fmaf(f[3], bf16_hi(v.y), s);
  s = fmaf(f[4], bf16_lo(v.z), s);
  s = fmaf(f[5], bf16_hi(v.z), s);
  s = fmaf(f[6], bf16_lo(v.w), s);
  s = fmaf(f[7], bf16_hi(v.w), s);
  return s;
}

// Score candidate rows [lo, lo+n) of Kc for this problem into keys[0, n).
// A half-warp scores 8 rows per step (8 x 16-byte loads in flight per lane).
__device__ void score_rows(const uint16_t *kc_bg, const float *fs, int nf, int lo, int n,
                           uint32_t *keys) {
  constexpr int kRows = 8;
  constexpr int kStep = (kSelThreads / 16) * kRows;  // rows per CTA step
  const int hw = threadIdx.x >> 4, hl = threadIdx.x & 15;
  const uint16_t *base = kc_bg + hl * 8;
#pragma unroll 1
  for (int r0 = 0; r0 < n; r0 += kStep) {
    const int row0 = r0 + hw * kRows;
    uint4 v[kRows];
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
      const int e = row0 + u;
      v[u] = e < n ? ldg_stream(base + (long long)(lo + e) * kD) : make_uint4(0, 0, 0, 0);
    }
    float part[kRows];
#pragma unroll
    for (int u = 0; u < kRows; ++u) part[u] = 0.f;
#pragma unroll 1
    for (int f = 0; f < nf; ++f) {
      float fv[8];
      const float4 a = *reinterpret_cast<const float4 *>(fs + f * kD + hl * 8);
      const float4 b = *reinterpret_cast<const float4 *>(fs + f * kD + hl * 8 + 4);
      fv[0] = a.x; fv[1] = a.y; fv[2] = a.z; fv[3] = a.w;
      fv[4] = b.x; fv[5] = b.y; fv[6] = b.z; fv[7] = b.w;
#pragma unroll
      for (int u = 0; u < kRows; ++u) part[u] += dot8(fv, v[u]);
    }
    const float s = transpose_reduce8x16(part, hl);
    const int e = row0 + (hl >> 1);
    if ((hl & 1) == 0 && e < n) keys[e] = orderable_key(s);
  }
}

__global__ void __launch_bounds__(kSelThreads, 2) select_kernel(SelArgs a) {
  extern __shared__ __align__(16) uint32_t dyn[];
  __shared__ __align__(16) float fs[kMaxNf * kD];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t bc[2];
  __shared__ uint32_t scan_tmp[33];
  __shared__ int s_last;

  // problems are laid out chunk-fastest so a problem's chunks run together
  // and its merge overlaps the streaming of later problems
  const long long prob = blockIdx.x / a.n_chunks;
  const int chunk = (int)(blockIdx.x - prob * a.n_chunks);
  const int g = (int)(prob % a.G);
  const long long bi = prob / a.G;
  const int i = (int)(bi % a.nq);
  const long long b = bi / a.nq;
  const BlockParts bp = block_parts(a.q_start + i, kBlk, a.n_init, a.n_local);
  const int ncand = bp.cand_hi - bp.cand_lo;
  int32_t *out = a.idx + prob * a.S;

  if (ncand <= a.k || a.k == 0) {  // nothing to rank: every candidate, or none, is kept
    if (chunk == 0) write_set(out, bp, min(ncand, a.k), a.S, true);
    return;
  }

  // Forecast vector(s) of this problem -> fp32 in shared memory
  const uint16_t *f = a.F + (bi * a.G + g) * (long long)a.nf * kD;
  for (int t = threadIdx.x; t < a.nf * kD; t += kSelThreads)
    fs[t] = __uint_as_float(((uint32_t)f[t]) << 16);
  __syncthreads();

  uint32_t *keys = dyn;
  const int lo = bp.cand_lo + chunk * a.CH;
  const int n = max(0, min(bp.cand_hi, lo + a.CH) - lo);
  const uint16_t *kc_bg = a.kc + (b * a.G + g) * (long long)a.NB * kD;
  score_rows(kc_bg, fs, a.nf, lo, n, keys);
  __syncthreads();

  uint32_t tau = 0;
  int need = 0;
  int32_t *top = out + bp.init_hi;

  if (a.n_chunks == 1) {  // n == ncand > k: rank in shared memory
    radix_threshold(keys, n, a.k, hist, bc, tau, need);
    const int ntop = compact_kept(
        keys, n, a.CH / kSelThreads, tau, need, scan_tmp, [&](int e) { return bp.cand_lo + e; },
        [&](int pos, uint32_t, int id) { top[pos] = id; });
    write_set(out, bp, ntop, a.S, false);
    return;
  }

  // ---- chunk scores -> workspace; the last chunk to finish ranks them all ----
  uint32_t *pkeys = a.cand_key + prob * (long long)a.cap;
  for (int e = threadIdx.x; e < n; e += kSelThreads) pkeys[chunk * a.CH + e] = keys[e];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned t = atomicAdd(&a.counters[prob], 1u);
    s_last = (t == (unsigned)(a.n_chunks - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int e = threadIdx.x; e < ncand; e += kSelThreads) keys[e] = __ldcg(pkeys + e);
  __syncthreads();
  radix_threshold(keys, ncand, a.k, hist, bc, tau, need);
  const int E = (ncand + kSelThreads - 1) / kSelThreads;
  const int ntop = compact_kept(
      keys, ncand, E, tau, need, scan_tmp, [&](int e) { return bp.cand_lo + e; },
      [&](int pos, uint32_t, int id) { top[pos] = id; });
  write_set(out, bp, ntop, a.S, false);
  if (threadIdx.x == 0) a.counters[prob] = 0u;
}

}  // namespace

int env_int(const char *name) {
  const char *s = getenv(name);
  return s ? atoi(s) : 0;
}

// The plan depends on the shapes only (not on where the query chunk sits), so
// the workspace size is known before the call: chunking is sized for a query
// at the end of the sequence, the most candidates any query can have.
SelectPlan plan_select(const sparda_params &p, int nq, int nf) {
  (void)nf;
  SelectPlan pl{};
  pl.n_problems = (long long)p.B * nq * p.G;
  const BlockParts bp = block_parts(p.T - 1, kBlk, p.n_init, p.n_local);
  pl.ncand_max = bp.cand_hi - bp.cand_lo;
  pl.CH = kSelThreads;
  pl.n_chunks = 1;
  pl.kc = 0;
  pl.ws_bytes = 0;
  if (pl.ncand_max <= p.k || p.k == 0 || pl.n_problems == 0) return pl;

  const int forced = env_int("SPARDA_SELECT_CHUNK");
  int CH;
  if (forced > 0) {
    CH = std::max(kSelThreads, (forced / kSelThreads) * kSelThreads);
  } else {
    // short-lived streaming CTAs: about 512 blocks (128 KB of Kc) each, but
    // one chunk per problem once there are plenty of problems (prefill)
    CH = 512;
    if (pl.n_problems >= 8LL * 148) CH = kMaxCand;
  }
  if (CH >= pl.ncand_max) CH = std::min(kMaxCand, (int)ceil_div_ll(pl.ncand_max, kSelThreads) * kSelThreads);
  pl.CH = CH;
  pl.n_chunks = (int)ceil_div_ll(pl.ncand_max, CH);
  if (pl.n_chunks > 1) {
    pl.kc = pl.ncand_max;  // every candidate's key is kept for the final rank
    size_t off = ((size_t)pl.n_problems * 4 + 255) & ~(size_t)255;      // counters
    off += (((size_t)pl.n_problems * pl.n_chunks * CH * 4) + 255) & ~(size_t)255;  // keys
    pl.ws_bytes = off;
  }
  return pl;
}

int select_supported(const SelectPlan &pl) {
  if (pl.CH > kMaxCand) return 0;
  if (pl.ncand_max > kMaxCand) return 0;
  return 1;
}

cudaError_t launch_select(const sparda_params &p, const SelectPlan &pl, const uint16_t *F, int nq,
                          int nf, int q_start, const uint16_t *kc, int32_t *idx, void *ws,
                          cudaStream_t stream) {
  if (pl.n_problems == 0) return cudaSuccess;
  SelArgs a;
  a.F = F;
  a.kc = kc;
  a.idx = idx;
  a.nq = nq;
  a.G = p.G;
  a.nf = nf;
  a.NB = (p.T + kBlk - 1) / kBlk;
  a.k = p.k;
  a.n_init = p.n_init;
  a.n_local = p.n_local;
  a.q_start = q_start;
  a.S = p.k + p.n_init + p.n_local;
  a.CH = pl.CH;
  a.n_chunks = pl.n_chunks;
  a.cap = pl.n_chunks * pl.CH;  // key slots per problem in the workspace
  a.counters = nullptr;
  a.cand_key = nullptr;
  size_t smem = (size_t)pl.CH * 4;
  if (pl.n_chunks > 1) {
    char *w = static_cast<char *>(ws);
    a.counters = reinterpret_cast<uint32_t *>(w);
    w += ((size_t)pl.n_problems * 4 + 255) & ~(size_t)255;
    a.cand_key = reinterpret_cast<uint32_t *>(w);
    smem = (size_t)std::max(pl.CH, pl.ncand_max) * 4;
  }
  if (smem > 48 * 1024) {  // raised once per device to the largest size used
    static size_t raised[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (raised[dev] < smem) {
      cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
      raised[dev] = smem;
    }
  }
  const long long grid = pl.n_problems * pl.n_chunks;
  select_kernel<<<(unsigned)grid, kSelThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace sparda
