// select_dev.cuh -- device pieces of the Forecast block selection on the
// block grid: the work of one (problem, chunk) item, and the slot-cache step
// the cached decode selection runs once a (b, g)'s set is written.
//
// Pages cited: [p4 <section>] = the article "SparDA: a fourth projection that
// lets sparse attention prefetch its own KV cache" (ai.thesatyajit.com).
// [p4 "The fourth projection", Eq. 4]: B_{l+1} = B_init U B_local U
//   f_top(F_l Kc_{l+1}^T, k); [p4 "One Forecast head per GQA group"].
//
// Everything here runs on kSelThreads = 256 threads and synchronises them
// with named barrier 3.
#pragma once

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "rank.cuh"

namespace sparda {
namespace {

// barrier among the 256 threads that run the selection
__device__ __forceinline__ void sel_sync() { asm volatile("bar.sync 3, 256;" ::: "memory"); }
__device__ __forceinline__ bool sel_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 3, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

constexpr int kSelThreads = 256;
constexpr int kMaxCand = 24576;   // candidates one problem may have (keys fit in shared memory)

struct SelArgs {
  const int32_t *seq_len;  // optional per-sequence lengths (decode: nq = 1)
  const uint16_t *F;
  const uint16_t *kc;
  int32_t *idx;
  uint32_t *counters;   // one ticket per problem (multi-chunk only)
  uint32_t *failed;     // one flag per problem: a chunk's copy never landed (multi-chunk only)
  uint32_t *cand_key;   // [problem][cap] score keys (multi-chunk only)
  int32_t *status;      // optional device status word
  int nq, G, nf, NB, k, n_init, n_local, q_start, S, T;
  int CH, n_chunks, cap;
  int NBf;       // window grid: blocks the key map covers (all three inner windows present)
  int old_rank;  // 1: always the binned threshold search
  SelCache cc;   // the cached decode selection's slot cache (cc.C == 0: none)
};

// ---------------------------------------------------------------------------
// block-wide helpers (blockDim.x == kSelThreads)
// ---------------------------------------------------------------------------

// ---------------------------------------------------------------------------
// exact k-th largest key
// ---------------------------------------------------------------------------
// Every pass below splits the current members -- the keys inside one
// contiguous key interval, all keys at first -- into 256 bins by a bin
// function that is monotone in the key, so the keys of one bin again form an
// interval and equal keys share a bin.  The bin that holds the wanted rank
// becomes the next members.  The first pass bins linearly in score value
// (for the usual bell-shaped scores the wanted bin then holds a handful of
// keys); later passes bin linearly in key space, which cuts the key range
// about 256-fold per pass, so at most six more passes reach a single key.
// Once 32 or fewer members remain, one warp ranks them exactly.  A pass costs
// four block barriers and a fixed number of conflict-free shared-memory
// reads per thread; no step depends on another thread's atomic result.
struct RankSmem {
  uint32_t hist[256];
  uint32_t wmin[kSelThreads / 32], wmax[kSelThreads / 32], wsum[kSelThreads / 32];
  uint32_t list[32];
  uint32_t units[64];      // packed per-(round row, warp) counts in compaction
  uint32_t bstar, rem, cnt, n_list, tau, need, carry;
};

// The k-th largest of keys[0, n) (tau) and how many keys equal to it are
// kept (need); 1 <= k < n.
__device__ void find_threshold(const uint32_t *keys, int n, int k, RankSmem &sm, uint32_t &tau,
                               int &need) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int nw = kSelThreads / 32;
  Members mem{};
  mem.all = true;
  uint32_t rem = (uint32_t)k, m = (uint32_t)n;
#pragma unroll 1
  for (int pass = 0; pass < 12; ++pass) {
    if (m <= 32u) {
      // ---- exact rank of the last few members by one warp ----
      if (tid == 0) sm.n_list = 0;
      sel_sync();
      for (int e = tid; e < n; e += kSelThreads) {
        const uint32_t u = keys[e];
        if (mem.has(u)) {
          const uint32_t slot = atomicAdd(&sm.n_list, 1u);
          if (slot < 32u) sm.list[slot] = u;
        }
      }
      sel_sync();
      if (warp == 0) {
        const uint32_t cnt = min(sm.n_list, 32u);
        const uint32_t x = (uint32_t)lane < cnt ? sm.list[lane] : 0u;
        uint32_t gt = 0, ge = 0;
        for (uint32_t j = 0; j < cnt; ++j) {
          const uint32_t y = sm.list[j];
          gt += y > x;
          ge += y >= x;
        }
        if ((uint32_t)lane < cnt && gt < rem && ge >= rem) {
          sm.tau = x;  // every lane holding this key writes the same values
          sm.need = rem - gt;
        }
      }
      sel_sync();
      tau = sm.tau;
      need = (int)sm.need;
      return;
    }
    // ---- key range of the members ----
    uint32_t umin = 0xFFFFFFFFu, umax = 0u;
    for (int e = tid; e < n; e += kSelThreads) {
      const uint32_t u = keys[e];
      if (mem.has(u)) {
        umin = min(umin, u);
        umax = max(umax, u);
      }
    }
    umin = __reduce_min_sync(0xffffffffu, umin);
    umax = __reduce_max_sync(0xffffffffu, umax);
    if (lane == 0) {
      sm.wmin[warp] = umin;
      sm.wmax[warp] = umax;
    }
    sm.hist[tid] = 0u;  // kSelThreads == 256 bins
    sel_sync();
#pragma unroll
    for (int w = 0; w < nw; ++w) {
      umin = min(umin, sm.wmin[w]);
      umax = max(umax, sm.wmax[w]);
    }
    if (umin == umax) {  // the members are all one key
      tau = umin;
      need = (int)rem;
      sel_sync();  // wmin / wmax are rewritten by nobody after this
      return;
    }
    // ---- bins over the members ----
    const Members nx = make_bins(pass, umin, umax);
    for (int e = tid; e < n; e += kSelThreads) {
      const uint32_t u = keys[e];
      if (mem.has(u)) atomicAdd(&sm.hist[nx.bin(u)], 1u);
    }
    sel_sync();
    // ---- the bin holding rank `rem` from the top: suffix sums over bins ----
    const uint32_t h = sm.hist[tid];
    uint32_t suf = h;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += t;
    }
    if (lane == 0) sm.wsum[warp] = suf;
    sel_sync();
#pragma unroll
    for (int w = 0; w < nw; ++w)
      if (w > warp) suf += sm.wsum[w];
    if (suf >= rem && suf - h < rem) {
      sm.bstar = (uint32_t)tid;
      sm.rem = rem - (suf - h);
      sm.cnt = h;
    }
    sel_sync();
    mem = nx;
    mem.b = sm.bstar;
    rem = sm.rem;
    m = sm.cnt;
  }
  // not reached: the key range is a single key after at most seven passes
  tau = 0xFFFFFFFFu;
  need = 0;
}

// The same threshold (tau, need) for k <= 64 and n <= 2048, with four block
// barriers instead of a dozen: every warp sorts its 256 keys in registers
// (a bitonic network, element q = 32*i + lane in register i, so partners
// closer than 32 are a shuffle away and farther ones sit in the lane's own
// registers), keeps its 64 largest, and three rounds of pairwise merges
// reduce the 8 lists to the 64 largest keys of all.  tau is the k-th of
// them and need counts how many keys equal to tau are kept; the
// compaction then picks exactly the same entries as after find_threshold.
// scratch: 1024 words of shared memory no one else is using.
constexpr int kTopkMaxK = 64, kTopkMaxN = 8 * kSelThreads;

__device__ __forceinline__ void cmp_swap_up(uint32_t &lo, uint32_t &hi, bool up) {
  const uint32_t a = min(lo, hi), b = max(lo, hi);
  lo = up ? a : b;
  hi = up ? b : a;
}

// Sort m*32 keys held as v[i] (element 32*i + lane) ascending within runs of
// `run` elements, the runs alternating direction as a bitonic network wants
// (ascending where (q & run) == 0); run == m*32 gives one ascending run.
template <int M>
__device__ __forceinline__ void bitonic_warp(uint32_t (&v)[M], int lane, int k_from, int k_to) {
#pragma unroll
  for (int kk = k_from; kk <= k_to; kk <<= 1) {
#pragma unroll
    for (int j = kk >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
        const int r = j >> 5;
#pragma unroll
        for (int i = 0; i < M; ++i) {
          if (i & r) continue;
          const int q = 32 * i + lane;
          cmp_swap_up(v[i], v[i | r], (q & kk) == 0);
        }
      } else {
#pragma unroll
        for (int i = 0; i < M; ++i) {
          const int q = 32 * i + lane;
          const uint32_t o = __shfl_xor_sync(0xffffffffu, v[i], j);
          const bool up = (q & kk) == 0, lower = (lane & j) == 0;
          v[i] = (up == lower) ? min(v[i], o) : max(v[i], o);
        }
      }
    }
  }
}

__device__ void find_threshold_topk(const uint32_t *keys, int n, int k, uint32_t *scratch,
                                    RankSmem &sm, uint32_t &tau, int &need) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  {  // each warp: its 256 keys sorted ascending, the largest 64 to scratch
    uint32_t v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = warp * 256 + 32 * i + lane;
      v[i] = e < n ? keys[e] : 0u;  // 0 sorts below every finite score's key
    }
    bitonic_warp<8>(v, lane, 2, 256);
    scratch[warp * 64 + lane] = v[6];
    scratch[warp * 64 + 32 + lane] = v[7];
  }
  sel_sync();
  // merges: lists a and b (ascending) -> the 64 largest of both, ascending:
  // c[x] = max(a[x], b[63 - x]) is bitonic and holds them, then one merge.
  // Rounds read one half of the scratch and write the other.
  uint32_t *src = scratch, *dst = scratch + 512;
#pragma unroll 1
  for (int lists = 8; lists > 1; lists >>= 1) {
    if (warp < lists / 2) {
      const uint32_t *a = src + (2 * warp) * 64, *b = src + (2 * warp + 1) * 64;
      uint32_t c[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int x = 32 * i + lane;
        c[i] = max(a[x], b[63 - x]);
      }
      bitonic_warp<2>(c, lane, 64, 64);
      dst[warp * 64 + lane] = c[0];  // list `warp` of the next round
      dst[warp * 64 + 32 + lane] = c[1];
    }
    sel_sync();
    uint32_t *t = src;
    src = dst;
    dst = t;
  }
  if (warp == 0) {
    const uint32_t x0 = src[lane], x1 = src[32 + lane];  // ascending, x1 holds 32..63
    const int pos = 64 - k;  // the k-th largest
    const uint32_t t = src[pos];
    const int gt = __popc(__ballot_sync(0xffffffffu, x0 > t)) + __popc(__ballot_sync(0xffffffffu, x1 > t));
    if (lane == 0) {
      sm.tau = t;
      sm.need = (uint32_t)(k - gt);
    }
  }
  sel_sync();
  tau = sm.tau;
  need = (int)sm.need;
}

// Keep keys > tau plus the first `need` keys == tau (in entry order), in
// entry order: out(pos, e) for each kept entry e, pos < limit.  Entries are
// visited 32 consecutive ones per warp step; the position of each kept entry
// comes from ballots inside the warp plus one block scan of per-warp counts
// per round of 8 x 256 entries.  Returns the number kept.
template <class Out>
__device__ int compact_kept(const uint32_t *keys, int n, uint32_t tau, int need, int limit,
                            RankSmem &sm, Out out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t carry = 0;  // packed (gt << 16 | eq) counts of earlier rounds
#pragma unroll 1
  for (int base = 0; base < n; base += 8 * kSelThreads) {
    uint32_t bgt[8], beq[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = base + i * kSelThreads + tid;
      const uint32_t u = e < n ? keys[e] : 0u;
      bgt[i] = __ballot_sync(0xffffffffu, e < n && u > tau);
      beq[i] = __ballot_sync(0xffffffffu, e < n && u == tau);
      if (lane == 0) sm.units[i * 8 + warp] = ((uint32_t)__popc(bgt[i]) << 16) | (uint32_t)__popc(beq[i]);
    }
    sel_sync();
    if (warp == 0) {  // exclusive scan of the 64 unit counts, two per lane
      const uint32_t a0 = sm.units[2 * lane], a1 = sm.units[2 * lane + 1];
      const uint32_t s = a0 + a1;
      uint32_t x = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
      }
      const uint32_t ex = carry + x - s;
      sm.units[2 * lane] = ex;
      sm.units[2 * lane + 1] = ex + a0;
      if (lane == 31) sm.carry = carry + x;
    }
    sel_sync();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t pre = sm.units[i * 8 + warp];
      const uint32_t gt_b = (pre >> 16) + (uint32_t)__popc(bgt[i] & lt);
      const uint32_t eq_b = (pre & 0xFFFFu) + (uint32_t)__popc(beq[i] & lt);
      const bool gt = (bgt[i] >> lane) & 1u, eq = (beq[i] >> lane) & 1u;
      if (gt || (eq && eq_b < (uint32_t)need)) {
        const uint32_t pos = gt_b + min(eq_b, (uint32_t)need);
        if (pos < (uint32_t)limit) out((int)pos, base + i * kSelThreads + tid);
      }
    }
    carry = sm.carry;
    sel_sync();  // units / carry are rewritten by the next round
  }
  return min(limit, (int)((carry >> 16) + min(carry & 0xFFFFu, (uint32_t)need)));
}

// A block-list entry, stored with an L2 evict-last hint: the attention that
// reads the list next streams hundreds of MB through L2 before it does, and
// the list's 34 KB (B = 16) should still be there.
__device__ __forceinline__ void st_list(int32_t *p, int v) {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  asm volatile("st.global.L2::cache_hint.b32 [%0], %1, %2;" ::"l"(p), "r"(v), "l"(pol) : "memory");
}

// init | top-k | local | -1 padding.  With `fill_top`, the top-k part is the
// first ntop candidates (every candidate is taken); otherwise it is written
// by the caller.  mirror (optional, shared memory): the entries written here
// are also stored there, at the same positions.
__device__ void write_set(int32_t *out, const BlockParts &bp, int ntop, int S, bool fill_top,
                          int32_t *mirror = nullptr) {
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
    st_list(out + s, v);
    if (mirror) mirror[s] = v;
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
// The rows (contiguous, 256 B each) are streamed by the bulk-copy engine in
// 128-row (32 KB) pieces through a kRing-deep shared-memory ring, so up to
// 96 KB per CTA are in flight with no register cost; each half-warp scores 8
// rows per piece from shared memory.  Returns false if a copy never landed
// (bounded wait), in which case the keys are not valid.
constexpr int kPieceRows = 128;
constexpr int kPieceBytes = kPieceRows * kD * 2;
constexpr int kRing = 3;  // pieces in flight (the selection kernel; the attention kernel's tail uses 2)

template <int RING = kRing>
__device__ __forceinline__ void issue_piece(const uint16_t *kc_bg, int lo, int n, int pc,
                                            uint8_t *ring, uint64_t *bars) {
  const int rows = min(kPieceRows, n - pc * kPieceRows);
  uint64_t *bar = &bars[pc % RING];
  mbar_arrive_expect_tx(bar, (uint32_t)rows * kD * 2);
  for (int r0 = 0; r0 < rows; r0 += 32)
    bulk_g2s(ring + (pc % RING) * kPieceBytes + r0 * kD * 2,
             kc_bg + (long long)(lo + pc * kPieceRows + r0) * kD,
             (uint32_t)min(32, rows - r0) * kD * 2, bar);
}

// thread 0, right after the barriers are initialised: the first pieces go
// out before anything else is loaded
template <int RING = kRing>
__device__ __forceinline__ void prime_ring(const uint16_t *kc_bg, int lo, int n, uint8_t *ring,
                                           uint64_t *bars) {
  const int n_pc = (n + kPieceRows - 1) / kPieceRows;
  for (int pc = 0; pc < min(RING, n_pc); ++pc) issue_piece<RING>(kc_bg, lo, n, pc, ring, bars);
}

// Block grid: key row r of the chunk scores block lo + r.
template <int RING = kRing>
__device__ bool score_rows(const uint16_t *kc_bg, const float *fs, int nf, int lo, int n,
                           uint32_t *keys, uint8_t *ring, uint64_t *bars) {
  const int hw = threadIdx.x >> 4, hl = threadIdx.x & 15;
  const int n_pc = (n + kPieceRows - 1) / kPieceRows;
  // the first pieces were issued by the caller's thread 0 right after the
  // barriers were initialised; the rest are refills
  bool ok = true;
#pragma unroll 1
  for (int pc = 0; pc < n_pc; ++pc) {
    const bool landed = mbar_wait_bounded(&bars[pc % RING], (uint32_t)((pc / RING) & 1));
    if (sel_sync_or(!landed)) {
      ok = false;
      // let copies still in flight land (bounded) before the ring is released
      if (threadIdx.x == 0)
        for (int q = pc; q < min(n_pc, pc + RING); ++q)
          (void)mbar_wait_bounded(&bars[q % RING], (uint32_t)((q / RING) & 1));
      sel_sync();
      break;
    }
    const int rows = min(kPieceRows, n - pc * kPieceRows);
    const uint8_t *piece = ring + (pc % RING) * kPieceBytes;
    const int row0 = hw * 8;
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      v[u] = row0 + u < rows ? *reinterpret_cast<const uint4 *>(piece + (row0 + u) * (kD * 2) + hl * 16)
                             : make_uint4(0, 0, 0, 0);
    float part[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) part[u] = 0.f;
#pragma unroll 1
    for (int f = 0; f < nf; ++f) {
      float fv[8];
      const float4 a = *reinterpret_cast<const float4 *>(fs + f * kD + hl * 8);
      const float4 b = *reinterpret_cast<const float4 *>(fs + f * kD + hl * 8 + 4);
      fv[0] = a.x; fv[1] = a.y; fv[2] = a.z; fv[3] = a.w;
      fv[4] = b.x; fv[5] = b.y; fv[6] = b.z; fv[7] = b.w;
#pragma unroll
      for (int u = 0; u < 8; ++u) part[u] += dot8(fv, v[u]);
    }
    const float sc = transpose_reduce8x16(part, hl);
    const int r = row0 + (hl >> 1);
    if ((hl & 1) == 0 && r < rows) keys[pc * kPieceRows + r] = orderable_key(sc);
    sel_sync();  // piece consumed by every half-warp
    if (threadIdx.x == 0 && pc + RING < n_pc) issue_piece<RING>(kc_bg, lo, n, pc + RING, ring, bars);
  }
  return ok;
}


// ---------------------------------------------------------------------------
// slot cache step of the cached decode selection
// ---------------------------------------------------------------------------
// [p4 "The fourth projection", Algorithm 2]: layer l+1's blocks come from
// CPU pinned memory while layer l computes.  The policy (the pages give
// none) is that of the plan kernel: a selected block some slot holds is a
// hit and keeps the slot; every other valid entry, in list order, takes the
// next slot past the clock hand that holds none of this step's blocks, and
// the hand moves one further.  Here the block that wrote a (b, g)'s set plans
// it and copies its misses, so the results equal those of the plan and
// gather calls made after the selection.

// The ring, idle once a set is written, holds the step's state (words):
// [0, 1024) the ranking's scratch | the list [S] (stored as it is written) |
// slot map [C] and hand [1] (loaded while the set is ranked) | slot of each
// entry [S] | lowest slot holding each entry's block [S] | slots in use
// (bits) | entries to copy [S] | their count [1]
__host__ __device__ constexpr long long cache_step_words(int C, int S) {
  return 1024LL + 4LL * S + C + (C + 31) / 32 + 2;
}

struct CacheSmem {
  int32_t *ids, *blk, *hand, *ph, *hit;
  uint32_t *used;
  int32_t *miss, *n_miss;
};

__device__ __forceinline__ CacheSmem cache_smem(uint8_t *ring, int C, int S) {
  CacheSmem cs;
  cs.ids = reinterpret_cast<int32_t *>(ring) + 1024;
  cs.blk = cs.ids + S;
  cs.hand = cs.blk + C;
  cs.ph = cs.hand + 1;
  cs.hit = cs.ph + S;
  cs.used = reinterpret_cast<uint32_t *>(cs.hit + S);
  cs.miss = reinterpret_cast<int32_t *>(cs.used + (C + 31) / 32);
  cs.n_miss = cs.miss + S;
  return cs;
}

__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

constexpr int kPlanMissMark = -2;
constexpr int kHitNone = 0x7fffffff;

// Start loading the pair's slot map and hand into the ring (asynchronous
// copies, waited for by cache_step), once the block knows it writes the set.
__device__ void cache_load_state(const SelArgs &a, long long pair, uint8_t *ring) {
  const CacheSmem cs = cache_smem(ring, a.cc.C, a.S);
  const int32_t *bo = a.cc.block_of + pair * a.cc.C;
  for (int c = threadIdx.x; c < a.cc.C; c += kSelThreads) cp_async4(cs.blk + c, bo + c);
  if (threadIdx.x == 0) cp_async4(cs.hand, a.cc.hand + pair);
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// An empty set (every entry -1): nothing is held or fetched, and the hand is
// only brought into range, as the plan leaves it.
__device__ void cache_step_empty(const SelArgs &a, long long pair) {
  const SelCache &cc = a.cc;
  for (int s = threadIdx.x; s < a.S; s += kSelThreads) {
    cc.phys[pair * a.S + s] = -1;
    cc.fetch[pair * a.S + s] = 0;
  }
  if (threadIdx.x == 0) {
    const int h = cc.hand[pair];
    if (h < 0 || h >= cc.C) cc.hand[pair] = 0;
  }
}

// The set this block has just written (ascending block ids, then -1
// padding; its entries also in cs.ids), after cache_load_state: plan it
// against the pair's C slots, write the plan's outputs and copy every miss
// from the mapped host blocks.  The list is sorted, so each slot finds the
// entry of its block by binary search (entries of -1 compare above every
// block id); a block held by several slots hits the lowest of them, as in
// the plan kernel.
__device__ void cache_step(const SelArgs &a, long long pair, uint8_t *ring) {
  const SelCache &cc = a.cc;
  const int tid = threadIdx.x, lane = tid & 31;
  const int C = cc.C, S = a.S, words = (C + 31) / 32;
  const CacheSmem cs = cache_smem(ring, C, S);
  for (int s = tid; s < S; s += kSelThreads) cs.hit[s] = kHitNone;
  for (int w = tid; w < words; w += kSelThreads) cs.used[w] = 0u;
  asm volatile("cp.async.wait_all;" ::: "memory");
  sel_sync();
  // hits: every slot looks its block up in the list
  for (int c = tid; c < C; c += kSelThreads) {
    const int j = cs.blk[c];
    if (j < 0) continue;
    int lo = 0, hi = S;  // the first entry not below j
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      const int v = cs.ids[mid];
      if (v >= 0 && v < j) lo = mid + 1;
      else hi = mid;
    }
    if (lo < S && cs.ids[lo] == j) atomicMin(&cs.hit[lo], c);
  }
  sel_sync();
  // one warp: the hits' slots marked in use, then the misses, in list order,
  // placed by one lane (the policy is sequential), found 32 entries at a time
  if (tid < 32) {
    for (int s = lane; s < S; s += 32) {
      const int j = cs.ids[s];
      int p = -1;
      if (j >= a.NB) {
        flag_status(a.status, SPARDA_DEV_RANGE);
      } else if (j >= 0) {
        p = cs.hit[s];
        if (p != kHitNone) atomicOr(&cs.used[p >> 5], 1u << (p & 31));
        else p = kPlanMissMark;
      }
      cs.ph[s] = p;
    }
    __syncwarp();
    int h = *cs.hand;
    if (h < 0 || h >= C) h = 0;
    int nm = 0;
    for (int base = 0; base < S; base += 32) {
      const int s = base + lane;
      unsigned m = __ballot_sync(0xffffffffu, s < S && cs.ph[s] == kPlanMissMark);
      while (m) {
        const int s2 = base + __ffs(m) - 1;
        m &= m - 1;
        if (lane == 0) {
          int guard = 0;  // a free slot exists while C >= S; bounded all the same
          while (((cs.used[h >> 5] >> (h & 31)) & 1u) && guard < C) {
            h = (h + 1 == C) ? 0 : h + 1;
            ++guard;
          }
          if (guard >= C) {
            cs.ph[s2] = -1;
            flag_status(a.status, SPARDA_DEV_RANGE);
          } else {
            cs.blk[h] = cs.ids[s2];
            cc.block_of[pair * C + h] = cs.ids[s2];  // only the slots that change are written
            cs.used[h >> 5] |= 1u << (h & 31);
            cs.ph[s2] = C + h;
            cs.miss[nm++] = s2;
            h = (h + 1 == C) ? 0 : h + 1;
          }
        }
        __syncwarp();
      }
    }
    if (lane == 0) {
      cc.hand[pair] = h;
      *cs.n_miss = nm;
    }
  }
  sel_sync();
  for (int s = tid; s < S; s += kSelThreads) {
    const int p = cs.ph[s];
    cc.phys[pair * S + s] = p >= C ? p - C : p;
    cc.fetch[pair * S + s] = p >= C ? 1 : 0;
  }
  // the copies: 16-byte zero-copy loads of the mapped host blocks, two
  // blocks' loads in flight per thread ahead of their stores
  constexpr int kVec = 2 * kBlk * kD * 2 / 16;  // 16-byte vectors of a K|V block pair
  constexpr int kPer = kVec / kSelThreads;      // 8 per thread
  const long long blk_elems = 2LL * kBlk * kD;
  const int nm = *cs.n_miss;
  for (int q = 0; q < nm; q += 2) {
    const int nb = min(2, nm - q);
    uint4 v[2][kPer];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (t < nb) {
        const uint4 *src = reinterpret_cast<const uint4 *>(
            cc.host_kv + (pair * a.NB + cs.ids[cs.miss[q + t]]) * blk_elems);
#pragma unroll
        for (int u = 0; u < kPer; ++u) v[t][u] = ldg_plain(src + u * kSelThreads + tid);
      }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (t < nb) {
        uint4 *dst = reinterpret_cast<uint4 *>(
            cc.cache + (pair * C + (cs.ph[cs.miss[q + t]] - C)) * blk_elems);
#pragma unroll
        for (int u = 0; u < kPer; ++u) stg_stream(dst + u * kSelThreads + tid, v[t][u]);
      }
    }
  }
}

// Shared memory one selection item works in.
struct SelSmem {
  uint8_t *ring;        // RING pieces of 32 KB, 16-byte aligned
  float *fs;            // the scoring vector(s), nf x 128 fp32
  uint32_t *keys;       // the chunk's own keys (CH)
  uint32_t *rank_keys;  // every candidate's key, for the ranking of a multi-chunk problem
  uint32_t *scratch;    // 1024 words for the sorting-network threshold
  uint64_t *bars;       // RING mbarriers
  RankSmem *rs;
  int *flags;           // [0] this chunk ranks the problem, [1] a chunk of it failed
};

// One chunk of one problem on the block grid: problem = item / n_chunks
// (problems chunk-fastest, so a problem's chunks run together), the chunk's
// CH candidates streamed through the ring and scored; a single-chunk problem
// is ranked at once, otherwise the keys go to the workspace and the chunk
// that takes the problem's last ticket ranks every key of it.  Runs on
// threads 0-255; every branch is uniform over them.
template <int RING, bool CACHED>
__device__ void select_block_item(const SelArgs &a, long long item, const SelSmem &sm) {
  const int tid = threadIdx.x;
  const long long prob = item / a.n_chunks;
  const int chunk = (int)(item - prob * a.n_chunks);
  const int g = (int)(prob % a.G);
  const long long bi = prob / a.G;
  const int i = (int)(bi % a.nq);
  const long long b = bi / a.nq;
  int pos = a.q_start + i;
  int32_t *out = a.idx + prob * a.S;
  if (a.seq_len) {  // per-sequence lengths: the queries are the sequence's last nq tokens
    const int len = a.seq_len[b];
    if (len < a.nq || len > a.T) {  // an invalid length: an empty set
      if (chunk == 0) {
        for (int s2 = tid; s2 < a.S; s2 += kSelThreads) out[s2] = -1;
        if (tid == 0) flag_status(a.status, SPARDA_DEV_RANGE);
        if (CACHED) cache_step_empty(a, prob);
      }
      if (a.n_chunks > 1) {  // keep the ticket count of the problem right
        sel_sync();
        if (tid == 0) {
          const unsigned t = atomicAdd(&a.counters[prob], 1u);
          if (t == (unsigned)(a.n_chunks - 1)) a.counters[prob] = 0u;
        }
      }
      return;
    }
    pos = len - a.nq + i;
  }
  const BlockParts bp = block_parts(pos, kBlk, a.n_init, a.n_local);
  const int ncand = bp.cand_hi - bp.cand_lo;
  if (ncand <= a.k || a.k == 0) {  // nothing to rank: every candidate, or none, is kept
    if (chunk == 0) {
      if (CACHED) cache_load_state(a, prob, sm.ring);  // no copy was issued: the ring is free
      write_set(out, bp, min(ncand, a.k), a.S, true,
                CACHED ? cache_smem(sm.ring, a.cc.C, a.S).ids : nullptr);
      if (CACHED) cache_step(a, prob, sm.ring);
    }
    return;
  }
  const int lo = bp.cand_lo + chunk * a.CH;
  const int n = max(0, min(bp.cand_hi, lo + a.CH) - lo);
  const int pg = (int)(b * a.G + g);  // (sequence, group): the key tensor's problem index
  const uint16_t *kc_bg = a.kc + (long long)pg * a.NB * kD;
  if (tid == 0) {
    for (int q = 0; q < RING; ++q) mbar_init(&sm.bars[q], 1);
    fence_mbar_init();
    prime_ring<RING>(kc_bg, lo, n, sm.ring, sm.bars);
  }
  // Forecast vector(s) of this problem -> fp32 in shared memory
  const uint16_t *f = a.F + (bi * a.G + g) * (long long)a.nf * kD;
  for (int t = tid; t < a.nf * kD; t += kSelThreads) sm.fs[t] = __uint_as_float(((uint32_t)f[t]) << 16);
  sel_sync();
  const bool ok = score_rows<RING>(kc_bg, sm.fs, a.nf, lo, n, sm.keys, sm.ring, sm.bars);
  // a copy that never landed: the problem's set is reported empty rather
  // than wrong (by the last chunk, when there are several)
  if (!ok && tid == 0) flag_status(a.status, SPARDA_DEV_TIMEOUT);
  sel_sync();
  uint32_t tau = 0;
  int need = 0;
  int32_t *top = out + bp.init_hi;
  // the list's shared-memory copy (the slot cache only)
  int32_t *mirror = CACHED ? cache_smem(sm.ring, a.cc.C, a.S).ids : nullptr;
  if (a.n_chunks == 1) {  // n == ncand > k: rank in shared memory
    if (!ok) {  // a copy may still land in the ring: the empty step uses none of it
      for (int s2 = tid; s2 < a.S; s2 += kSelThreads) out[s2] = -1;
      if (CACHED) cache_step_empty(a, prob);
      return;
    }
    if (CACHED) cache_load_state(a, prob, sm.ring);  // every copy of this block landed
    if (a.k <= kTopkMaxK && n <= kTopkMaxN && !a.old_rank)
      find_threshold_topk(sm.keys, n, a.k, sm.scratch, *sm.rs, tau, need);
    else
      find_threshold(sm.keys, n, a.k, *sm.rs, tau, need);
    const int ntop = compact_kept(sm.keys, n, tau, need, a.k, *sm.rs, [&](int p2, int e) {
      st_list(top + p2, bp.cand_lo + e);
      if (CACHED) mirror[bp.init_hi + p2] = bp.cand_lo + e;
    });
    write_set(out, bp, ntop, a.S, false, mirror);
    if (CACHED) cache_step(a, prob, sm.ring);
    return;
  }
  // ---- chunk scores -> workspace; the last chunk to finish ranks them all.
  // A chunk whose copy never landed still takes its ticket (so the count
  // completes and the last chunk resets it) and raises the problem's flag ----
  uint32_t *pkeys = a.cand_key + prob * (long long)a.cap;
  if (ok)
    for (int e = tid; e < n; e += kSelThreads) pkeys[chunk * a.CH + e] = sm.keys[e];
  else if (tid == 0)
    a.failed[prob] = 1u;
  __threadfence();
  sel_sync();
  if (tid == 0) {
    const unsigned t = atomicAdd(&a.counters[prob], 1u);
    sm.flags[0] = (t == (unsigned)(a.n_chunks - 1));
  }
  sel_sync();
  if (!sm.flags[0]) return;
  __threadfence();
  if (tid == 0) sm.flags[1] = (int)__ldcg(a.failed + prob);
  sel_sync();
  if (sm.flags[1]) {
    for (int s2 = tid; s2 < a.S; s2 += kSelThreads) out[s2] = -1;
    if (tid == 0) {
      a.failed[prob] = 0u;
      a.counters[prob] = 0u;
    }
    if (CACHED) cache_step_empty(a, prob);
    return;
  }
  uint32_t *keys = sm.rank_keys;
  // this block's own copies all landed (else the problem failed): the ring is free
  if (CACHED) cache_load_state(a, prob, sm.ring);
  for (int e = tid; e < ncand; e += kSelThreads) keys[e] = __ldcg(pkeys + e);
  sel_sync();
  if (a.k <= kTopkMaxK && ncand <= kTopkMaxN && !a.old_rank)
    find_threshold_topk(keys, ncand, a.k, sm.scratch, *sm.rs, tau, need);
  else
    find_threshold(keys, ncand, a.k, *sm.rs, tau, need);
  const int ntop = compact_kept(keys, ncand, tau, need, a.k, *sm.rs, [&](int p2, int e) {
    st_list(top + p2, bp.cand_lo + e);
    if (CACHED) mirror[bp.init_hi + p2] = bp.cand_lo + e;
  });
  write_set(out, bp, ntop, a.S, false, mirror);
  if (tid == 0) a.counters[prob] = 0u;
  if (CACHED) cache_step(a, prob, sm.ring);
}


}  // namespace
}  // namespace sparda
