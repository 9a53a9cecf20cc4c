// select_prefill.cu -- Forecast block selection for a chunk of query tokens
// (prefill): every token of the chunk scores every candidate block of its
// sequence with its own Forecast vector and keeps the k best.
//
// Pages cited: [p4 <section>] = the article "SparDA: a fourth projection that
// lets sparse attention prefetch its own KV cache" (ai.thesatyajit.com);
// [p1 <section>] = the SparDA summary page at deepresearch2agi.pages.dev.
//
// [p4 "The fourth projection", Algorithm 1]: B_l = B_init U B_local U
//   top_k(F_prev @ K_compressed[l].T, k), per query token, each token with
//   its own causal candidate range;
// [p4 "One Forecast head per GQA group"]: one Forecast vector per group, raw
//   dot products, no softmax.
//
// Design (B200).  For one (sequence, group) the scores of a chunk are a
// dense product S = F_chunk Kc^T: 2048 tokens x 2048 blocks x 128 dims, 34
// GFLOP over the 4 x 8 pairs of the benchmark chunk.  That is a tensor-core
// contraction, so it runs in two kernels:
//  1. prefill_scores_kernel -- one CTA per (pair, 128-token tile, 256-block
//     tile): TMA loads the F tile (4-D map: dims, group, token, sequence) and
//     the Kc tile (3-D map: dims, block, pair), one thread issues eight
//     tcgen05 MMAs (M = 128 tokens, N = 256 blocks, K = 16 each) into TMEM,
//     and the four warps read the 128 x 256 fp32 scores back (thread = token
//     row), turn them into orderable keys -- 0 outside the token's candidate
//     range -- and store them to the workspace, [pair][token][block].  Tiles
//     lying wholly after every row's candidates are skipped.
//  2. rank_rows_kernel -- one warp per (sequence, token, group) row.  For
//     k <= 64 and rows of 1024 to 2048 keys it first takes a threshold t0
//     that at least 64 keys pass (the least over the lanes of each lane's
//     second-largest key), lists the keys >= t0 (about 9 % of a row) and
//     ranks only those: one histogram, an exact rank of the threshold bin,
//     and a bitmap that puts the kept blocks in order.  Other rows, and rows
//     whose lists or ties that does not settle, take the same exact search as
//     the decode selection (a score-linear then key-linear 256-bin passes, an
//     exact rank of the last few candidates) with a per-warp histogram in
//     shared memory, then a ballot pass in block order that keeps every key
//     above the k-th plus the lowest-index ties.  The set is init U top-k U
//     local, written in ascending order.
// Every wait is bounded; a timeout sets SPARDA_DEV_TIMEOUT, frees TMEM and
// leaves the tile's keys unwritten.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "rank.cuh"
#include "tc.cuh"

namespace sparda {

namespace {

constexpr int kPTok = 128;      // token rows per score tile (MMA M)
constexpr int kPBlk = 256;      // block columns per score tile (MMA N)
constexpr int kPThreads = 128;  // four warps: TMEM lanes 0-127, thread = token row
constexpr int kPSmem = 32768 + 65536 + 1024;  // F tile | Kc tile | barriers
constexpr int kRWarps = 8;        // rows ranked per CTA (one warp each), binned search alone
constexpr int kRWarpsListed = 4;  // the same with the listed threshold (larger per-warp lists)

struct PScoreArgs {
  uint32_t *keys;      // [B*G][nq][ld]
  int32_t *status;
  int G, nq, NB, ld, q_start, n_init, n_local;
  int n_rows;          // key rows per (b, g): blocks, or windows (kPool = 4)
  const int32_t *seq_len;  // optional: the chunk is each sequence's last nq tokens
  int T;
};

// kPool = 1: one key row per block, tile column c is block j0 + c.  kPool = 4
// (window grid): columns are windows, four per block, and block j scores as
// the best of its windows 4j, 4j+1, 4j+2 (window 4j+3 straddles two blocks).
template <int kPool>
__global__ void __launch_bounds__(kPThreads) prefill_scores_kernel(
    const __grid_constant__ CUtensorMap mapF, const __grid_constant__ CUtensorMap mapKc,
    PScoreArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *opA = smem;            // [2 dim halves][128 tokens][64 dims], 32 KB
  uint8_t *opB = smem + 32768;    // [2 dim halves][256 blocks][64 dims], 64 KB
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 32768 + 65536);  // tma, mma
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int u = blockIdx.x, t = blockIdx.y, pair = blockIdx.z;
  const int b = pair / a.G, g = pair % a.G;
  const int i0 = t * kPTok;
  const int w0 = u * kPBlk;       // first key row (block or window) of the tile
  const int j0 = w0 / kPool;      // first block of the tile
  pdl_trigger();
  // with per-sequence lengths the chunk is the sequence's last nq tokens (the
  // length is read once the previous kernel is done); an invalid length
  // leaves the rows to the ranking kernel, which writes empty sets
  int qs = a.q_start, n_rows = a.n_rows;
  if (a.seq_len) {
    pdl_wait();
    const int len = a.seq_len[b];
    if (len < a.nq || len > a.T) return;
    qs = len - a.nq;
    if (kPool > 1) n_rows = window_count(len);
  }
  // the candidates of the tile's last row reach furthest
  const int i_last = min(a.nq, i0 + kPTok) - 1;
  const BlockParts bp_last = block_parts(qs + i_last, kBlk, a.n_init, a.n_local);
  if (j0 >= bp_last.cand_hi || j0 + kPBlk / kPool <= a.n_init) return;  // no candidate in the tile
  if (smem_addr(smem) & 1023u) {
    pdl_wait();
    if (tid == 0) flag_status(a.status, SPARDA_DEV_LAYOUT);
    return;
  }
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    tc::prefetch_map(&mapF);
    tc::prefetch_map(&mapKc);
  }
  if (warp == 0) tc::tmem_alloc(tmem_slot, 256);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();

  bool ok = true;
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], 32768 + 65536);
    tc::tma_load_4d(opA, &mapF, 0, g, i0, b, &bars[0]);
    tc::tma_load_4d(opA + 16384, &mapF, 64, g, i0, b, &bars[0]);
    tc::tma_load_3d(opB, &mapKc, 0, w0, pair, &bars[0]);
    tc::tma_load_3d(opB + 32768, &mapKc, 64, w0, pair, &bars[0]);
    ok = mbar_wait_bounded(&bars[0], 0);
    if (ok) {
      tc::fence_after_sync();
      constexpr uint32_t id = tc::idesc_bf16(kPTok, kPBlk, false, false);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        tc::mma_bf16(tmem, tc::sdesc(opA + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                     tc::sdesc(opB + (k >> 2) * 32768 + (k & 3) * 32, 16, 1024), id, k > 0);
      tc::mma_commit(&bars[1]);
    }
  }
  const bool tma_ok = __syncthreads_and(ok);
  if (tma_ok) ok = mbar_wait_bounded(&bars[1], 0);
  ok = __syncthreads_and(ok);
  if (!ok) {
    if (tid == 0) {
      flag_status(a.status, SPARDA_DEV_TIMEOUT);
      // give copies still in flight a bounded chance to land before the
      // shared memory is released
      if (!tma_ok) (void)mbar_wait_bounded(&bars[0], 0);
    }
  } else {
    tc::fence_after_sync();
    const int i = i0 + tid;  // this thread's token row (TMEM lane tid)
    const BlockParts bp = block_parts(qs + min(i, a.nq - 1), kBlk, a.n_init, a.n_local);
    uint32_t *row = a.keys + ((long long)pair * a.nq + i) * a.ld + j0;
    const uint32_t lane_sel = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
    for (int c = 0; c < kPBlk; c += 16) {
      float v[16];
      tc::tmem_ld16(tmem + lane_sel + c, v);  // warp-wide: every lane takes part
      if (kPool == 1) {
        if (j0 + c < a.ld) {
          // the warp's 32 rows x 16 keys go through shared memory (the A
          // operand's space, free once the products are done), so each store
          // writes whole 64-byte row pieces: 16-byte chunks rotated by row
          uint32_t kk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int j = j0 + c + e;
            kk[e] = (j >= bp.cand_lo && j < bp.cand_hi) ? orderable_key(v[e]) : 0u;
          }
          uint8_t *stg = opA + warp * 2048;  // [32 rows][64 bytes]
          const int rl = tid & 31;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4 *>(stg + rl * 64 + ((q ^ (rl & 3)) << 4)) =
                make_uint4(kk[4 * q], kk[4 * q + 1], kk[4 * q + 2], kk[4 * q + 3]);
          __syncwarp();
#pragma unroll
          for (int t2 = 0; t2 < 4; ++t2) {
            const int r2 = t2 * 8 + (rl >> 2), q2 = rl & 3;  // row of the warp, chunk
            const int i2 = i0 + warp * 32 + r2;
            const uint4 val = *reinterpret_cast<const uint4 *>(stg + r2 * 64 + ((q2 ^ (r2 & 3)) << 4));
            if (i2 < a.nq)
              reinterpret_cast<uint4 *>(a.keys + ((long long)pair * a.nq + i2) * a.ld + j0 + c)[q2] = val;
          }
          __syncwarp();  // the staging rows are rewritten by the next step
        }
      } else {
        // 16 window columns = 4 blocks; windows past the last one are masked
        if (i < a.nq) {
          uint32_t kk[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float m = -INFINITY;
#pragma unroll
            for (int e = 0; e < 3; ++e)
              if (w0 + c + 4 * q + e < n_rows) m = fmaxf(m, v[4 * q + e]);
            const int j = j0 + c / 4 + q;
            kk[q] = (j >= bp.cand_lo && j < bp.cand_hi) ? orderable_key(m) : 0u;
          }
          *reinterpret_cast<uint4 *>(row + c / 4) = make_uint4(kk[0], kk[1], kk[2], kk[3]);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// warp-level exact top-k of one row
// ---------------------------------------------------------------------------
constexpr int kListCap = 24;  // keys per lane the sampled threshold may list

struct WarpRankSmem {
  uint32_t hist[256];
  uint32_t list[32];
};

// the listed threshold's lists on top
struct WarpListSmem : WarpRankSmem {
  uint2 cand[kListCap + 1][32];  // per lane: (key, register q) of its keys >= t0; row
                                 // kListCap takes the writes past the cap
  uint32_t sel[64];              // kept entries: word q, bit lane = entry 32 q + lane
};

// the keys were written by the previous kernel: read-only for this one
__device__ __forceinline__ uint32_t ld_key(const uint32_t *p) { return __ldg(p); }

// The k-th largest of keys[0, n) and how many keys equal to it are kept;
// 1 <= k < n; one warp, no block barrier.
__device__ void warp_threshold(const uint32_t *keys, int n, int k, WarpRankSmem &sm,
                               uint32_t &tau, int &need) {
  const int lane = threadIdx.x & 31;
  Members mem{};
  mem.all = true;
  uint32_t rem = (uint32_t)k, m = (uint32_t)n;
#pragma unroll 1
  for (int pass = 0; pass < 12; ++pass) {
    if (m <= 32u) {
      // ---- exact rank of the last few members ----
      uint32_t cnt = 0;
#pragma unroll 1
      for (int base = 0; base < n; base += 32) {
        const int e = base + lane;
        const uint32_t u = e < n ? ld_key(keys + e) : 0u;
        const bool in = e < n && mem.has(u);
        const uint32_t bal = __ballot_sync(0xffffffffu, in);
        const uint32_t slot = cnt + __popc(bal & ((1u << lane) - 1u));
        if (in && slot < 32u) sm.list[slot] = u;
        cnt += __popc(bal);
      }
      __syncwarp();
      cnt = min(cnt, 32u);
      const uint32_t x = (uint32_t)lane < cnt ? sm.list[lane] : 0u;
      uint32_t gt = 0, ge = 0;
      for (uint32_t j = 0; j < cnt; ++j) {
        const uint32_t y = sm.list[j];
        gt += y > x;
        ge += y >= x;
      }
      const bool hit = (uint32_t)lane < cnt && gt < rem && ge >= rem;
      const uint32_t who = __ballot_sync(0xffffffffu, hit);
      const int src = who ? __ffs(who) - 1 : 0;
      tau = __shfl_sync(0xffffffffu, x, src);
      need = (int)(rem - __shfl_sync(0xffffffffu, gt, src));
      __syncwarp();
      return;
    }
    // ---- key range of the members ----
    uint32_t umin = 0xFFFFFFFFu, umax = 0u;
#pragma unroll 4
    for (int e = lane; e < n; e += 32) {
      const uint32_t u = ld_key(keys + e);
      if (mem.has(u)) {
        umin = min(umin, u);
        umax = max(umax, u);
      }
    }
    umin = __reduce_min_sync(0xffffffffu, umin);
    umax = __reduce_max_sync(0xffffffffu, umax);
    if (umin == umax) {
      tau = umin;
      need = (int)rem;
      return;
    }
    // ---- histogram over the next bins ----
    const Members nx = make_bins(pass, umin, umax);
#pragma unroll
    for (int q = 0; q < 8; ++q) sm.hist[lane * 8 + q] = 0u;
    __syncwarp();
#pragma unroll 4
    for (int e = lane; e < n; e += 32) {
      const uint32_t u = ld_key(keys + e);
      if (mem.has(u)) atomicAdd(&sm.hist[nx.bin(u)], 1u);
    }
    __syncwarp();
    // ---- the bin holding rank `rem` from the top ----
    uint32_t h[8], local = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      h[q] = sm.hist[lane * 8 + q];
      local += h[q];
    }
    uint32_t above = local;  // inclusive suffix over lanes, then exclusive
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_down_sync(0xffffffffu, above, o);
      if (lane + o < 32) above += v;
    }
    above -= local;  // keys in bins of higher lanes
    int bsel = -1;
    uint32_t rsel = 0, csel = 0;
#pragma unroll
    for (int q = 7; q >= 0; --q) {
      if (bsel < 0 && above + h[q] >= rem && above < rem) {
        bsel = lane * 8 + q;
        rsel = rem - above;
        csel = h[q];
      }
      above += h[q];
    }
    const uint32_t who = __ballot_sync(0xffffffffu, bsel >= 0);
    const int src = who ? __ffs(who) - 1 : 0;
    mem = nx;
    mem.b = (uint32_t)__shfl_sync(0xffffffffu, bsel, src);
    rem = __shfl_sync(0xffffffffu, rsel, src);
    m = __shfl_sync(0xffffffffu, csel, src);
    __syncwarp();
  }
  tau = 0xFFFFFFFFu;  // not reached: the range is a single key within seven passes
  need = 0;
}

// The smallest key u in [lo, hi] whose bin is at least b (hi when none is
// below it): bins are monotone in the key, so the warp splits [lo, hi] 32
// ways per round, each lane testing one cut (at most seven rounds).
__device__ __forceinline__ uint32_t first_key_with_bin(const Members &mem, uint32_t lo,
                                                       uint32_t hi, uint32_t b) {
  const int lane = threadIdx.x & 31;
#pragma unroll 1
  for (int round = 0; round < 10 && lo < hi; ++round) {
    const uint64_t span = (uint64_t)(hi - lo);
    const uint32_t cut = lo + (uint32_t)((span * (uint64_t)(lane + 1)) >> 5);  // lane 31: hi
    const uint32_t ok = __ballot_sync(0xffffffffu, mem.bin(cut) >= b);
    const int first = ok ? __ffs(ok) - 1 : 31;
    const uint32_t below = __shfl_sync(0xffffffffu, cut, first > 0 ? first - 1 : 0);
    const uint32_t at = __shfl_sync(0xffffffffu, cut, first);
    if (!ok) return hi;  // not reached: bin(hi) >= b for the bins searched here
    lo = first > 0 ? below + 1 : lo;
    hi = at;
  }
  return hi;
}

// The same search with the row held in registers: entry e = 32*q + lane is
// kv[q] (0 past the row's end; a valid key is never 0), m of them valid,
// umin / umax the smallest and largest valid key.  Each pass histograms the
// members in shared memory; once the bin holding the wanted rank has at most
// 32 members, its key interval is found by a 32-way search of the monotone
// bin function and the members are ranked exactly.  n_tau: the row's keys
// equal to tau.
template <int KPL>
__device__ void warp_threshold_reg(const uint32_t (&kv)[KPL], uint32_t m, uint32_t umin,
                                   uint32_t umax, int k, WarpRankSmem &sm, uint32_t &tau,
                                   int &need, int &n_tau) {
  const int lane = threadIdx.x & 31;
  uint32_t rem = (uint32_t)k;
  // the members: valid keys in [lo, hi].  lo >= umin >= 1, so with one
  // unsigned comparison of kv - lo against hi - lo an empty entry (0) wraps
  // past the interval
  uint32_t lo = umin, hi = umax;
#pragma unroll 1
  for (int pass = 0; pass < 12; ++pass) {
    const uint32_t width = hi - lo;
    if (m <= 32u || lo == hi) {
      // ---- exact rank of the last few members ----
      uint32_t cnt = 0;
#pragma unroll
      for (int q = 0; q < KPL; ++q) {
        const bool in = kv[q] - lo <= width;
        const uint32_t bal = __ballot_sync(0xffffffffu, in);
        const uint32_t slot = cnt + __popc(bal & ((1u << lane) - 1u));
        if (in && slot < 32u) sm.list[slot] = kv[q];
        cnt += __popc(bal);
      }
      __syncwarp();
      if (lo == hi) {  // every member equal
        tau = lo;
        need = (int)rem;
        n_tau = (int)cnt;
        return;
      }
      cnt = min(cnt, 32u);
      const uint32_t x = (uint32_t)lane < cnt ? sm.list[lane] : 0u;
      uint32_t gt = 0, ge = 0;
      for (uint32_t j = 0; j < cnt; ++j) {
        const uint32_t y = sm.list[j];
        gt += y > x;
        ge += y >= x;
      }
      const bool hit = (uint32_t)lane < cnt && gt < rem && ge >= rem;
      const uint32_t who = __ballot_sync(0xffffffffu, hit);
      const int src = who ? __ffs(who) - 1 : 0;
      tau = __shfl_sync(0xffffffffu, x, src);
      need = (int)(rem - __shfl_sync(0xffffffffu, gt, src));
      n_tau = (int)(__shfl_sync(0xffffffffu, ge - gt, src));
      __syncwarp();
      return;
    }
    // ---- histogram of the members over the next bins ----
    const Members nx = make_bins(pass, lo, hi);
#pragma unroll
    for (int q = 0; q < 8; ++q) sm.hist[lane * 8 + q] = 0u;
    __syncwarp();
#pragma unroll
    for (int q = 0; q < KPL; ++q)
      if (kv[q] - lo <= width) atomicAdd(&sm.hist[nx.bin(kv[q])], 1u);
    __syncwarp();
    // ---- the bin holding rank `rem` from the top ----
    uint32_t h[8], local = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      h[q] = sm.hist[lane * 8 + q];
      local += h[q];
    }
    uint32_t above = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_down_sync(0xffffffffu, above, o);
      if (lane + o < 32) above += v;
    }
    above -= local;
    int bsel = -1;
    uint32_t rsel = 0, csel = 0;
#pragma unroll
    for (int q = 7; q >= 0; --q) {
      if (bsel < 0 && above + h[q] >= rem && above < rem) {
        bsel = lane * 8 + q;
        rsel = rem - above;
        csel = h[q];
      }
      above += h[q];
    }
    const uint32_t who = __ballot_sync(0xffffffffu, bsel >= 0);
    const int src = who ? __ffs(who) - 1 : 0;
    const uint32_t b = (uint32_t)__shfl_sync(0xffffffffu, bsel, src);
    rem = __shfl_sync(0xffffffffu, rsel, src);
    m = __shfl_sync(0xffffffffu, csel, src);
    // the bin's key interval within [lo, hi]
    const uint32_t a = first_key_with_bin(nx, lo, hi, b);
    const uint32_t c = b >= 255u ? hi : first_key_with_bin(nx, lo, hi, b + 1);
    const bool c_in = b < 255u && nx.bin(c) > b;  // c is past the bin: its last key is c - 1
    lo = a;
    hi = c_in ? c - 1 : c;
    __syncwarp();
  }
  tau = 0xFFFFFFFFu;  // not reached: the range is a single key within a few passes
  need = 0;
  n_tau = 0;
}

constexpr int kRegKeys = 64;  // keys per lane held in registers (rows up to 2048)

// The row's top k from a sampled threshold, for k <= 64 and rows of 1024 to
// 2048 keys, each lane taking the entries e = 32 q + lane as in the register
// search above (0 past the row).  t0 is the smallest over the lanes of each
// lane's second-largest key, so every lane holds two keys >= t0 and at least
// 64 >= k keys pass it: the k-th largest key is >= t0, and so is every key
// the set keeps.  On scores of roughly one shape across the row a lane holds
// about six such keys of its 64 (more than kListCap = 24 in none of 3000
// modelled Gaussian rows; 16 would overflow in about 2 %).  Each lane lists its keys >= t0 in shared memory (list_keys_from),
// one histogram of the listed keys finds the bin of the k-th largest, its
// members are ranked exactly, and the kept entries are placed in block order
// through a bitmap (word q, bit lane) and its prefix counts
// (warp_topk_listed).  warp_topk_listed returns false, having written
// nothing, when a lane lists more than kListCap keys, the bin holds more than
// 32 keys, or only some of the keys equal to the k-th are kept (the lower
// block indices would have to win); the caller then runs the full search.

// c = the lane's keys >= t0 (t0 >= 1, so never an empty entry), read again
// from memory (L1 holds the row just read); only the first kListCap are
// stored
__device__ __forceinline__ int list_keys_from(const uint32_t *keys, int ncand, uint32_t t0,
                                              WarpListSmem &sm) {
  const int lane = threadIdx.x & 31;
  __builtin_assume(ncand >= 1024);  // the listed threshold takes rows of 1024 keys or more
  int c = 0;
#pragma unroll 8
  for (int q = 0; q < kRegKeys; ++q) {
    const int e = q * 32 + lane;
    const uint32_t u = e < ncand ? ld_key(keys + e) : 0u;
    if (u >= t0) {
      sm.cand[min(c, kListCap)][lane] = make_uint2(u, (uint32_t)q);
      ++c;
    }
  }
  return c;
}

__device__ bool warp_topk_listed(int c, uint32_t t0, uint32_t umax, int k, WarpListSmem &sm,
                                 int32_t *top, int cand_lo) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  if (__any_sync(0xffffffffu, c > kListCap)) return false;
  const int cmax = __reduce_max_sync(0xffffffffu, (uint32_t)c);
  // ---- one histogram of the listed keys, bins linear in score over [t0, umax] ----
  const Members nx = make_bins(0, t0, umax);
#pragma unroll
  for (int q = 0; q < 8; ++q) sm.hist[lane * 8 + q] = 0u;
  __syncwarp();
  for (int i = 0; i < c; ++i) atomicAdd(&sm.hist[nx.bin(sm.cand[i][lane].x)], 1u);
  __syncwarp();
  uint32_t h[8], local = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    h[q] = sm.hist[lane * 8 + q];
    local += h[q];
  }
  uint32_t above = local;  // keys in the bins of this lane and the lanes above it
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, above, o);
    if (lane + o < 32) above += v;
  }
  above -= local;
  const uint32_t rank = (uint32_t)k;
  int bsel = -1;
  uint32_t rsel = 0, csel = 0;
#pragma unroll
  for (int q = 7; q >= 0; --q) {
    if (bsel < 0 && above + h[q] >= rank && above < rank) {
      bsel = lane * 8 + q;
      rsel = rank - above;
      csel = h[q];
    }
    above += h[q];
  }
  const uint32_t who_b = __ballot_sync(0xffffffffu, bsel >= 0);
  const int src_b = who_b ? __ffs(who_b) - 1 : 0;
  const uint32_t b = (uint32_t)__shfl_sync(0xffffffffu, bsel, src_b);
  const uint32_t rem = __shfl_sync(0xffffffffu, rsel, src_b);
  const uint32_t m = __shfl_sync(0xffffffffu, csel, src_b);
  if (!who_b || m > 32u) return false;
  // ---- the bin's keys, ranked exactly ----
  uint32_t cnt = 0;
  for (int i = 0; i < cmax; ++i) {
    const uint32_t u = i < c ? sm.cand[i][lane].x : 0u;
    const bool in = i < c && nx.bin(u) == b;
    const uint32_t bal = __ballot_sync(0xffffffffu, in);
    if (in) sm.list[cnt + __popc(bal & lt)] = u;
    cnt += __popc(bal);
  }
  __syncwarp();
  const uint32_t x = (uint32_t)lane < cnt ? sm.list[lane] : 0u;
  uint32_t gt = 0, ge = 0;
  for (uint32_t j = 0; j < cnt; ++j) {
    const uint32_t y = sm.list[j];
    gt += y > x;
    ge += y >= x;
  }
  const bool hit = (uint32_t)lane < cnt && gt < rem && ge >= rem;
  const uint32_t who = __ballot_sync(0xffffffffu, hit);
  const int src = who ? __ffs(who) - 1 : 0;
  const uint32_t tau = __shfl_sync(0xffffffffu, x, src);
  const uint32_t need = rem - __shfl_sync(0xffffffffu, gt, src);
  const uint32_t n_tau = __shfl_sync(0xffffffffu, ge - gt, src);
  if (!who || need != n_tau) return false;
  // ---- exactly k listed keys are >= tau: place them in block order ----
  sm.sel[lane] = 0u;
  sm.sel[lane + 32] = 0u;
  __syncwarp();
  for (int i = 0; i < c; ++i) {
    const uint2 e = sm.cand[i][lane];
    if (e.x >= tau) atomicOr(&sm.sel[e.y], 1u << lane);
  }
  __syncwarp();
  const uint32_t w0 = sm.sel[2 * lane], w1 = sm.sel[2 * lane + 1];
  const uint32_t n0 = __popc(w0), n01 = n0 + __popc(w1);
  uint32_t incl = n01;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  sm.hist[2 * lane] = incl - n01;  // kept entries before word 2 lane
  sm.hist[2 * lane + 1] = incl - n01 + n0;
  __syncwarp();
  for (int i = 0; i < c; ++i) {
    const uint2 e = sm.cand[i][lane];
    if (e.x >= tau) top[sm.hist[e.y] + __popc(sm.sel[e.y] & lt)] = cand_lo + 32 * (int)e.y + lane;
  }
  __syncwarp();
  return true;
}

struct RankArgs {
  const uint32_t *keys;  // [B*G][nq][ld]
  int32_t *idx;          // [B][nq][G][S]
  long long rows;        // B * nq * G
  int G, nq, ld, k, n_init, n_local, q_start, S;
  const int32_t *seq_len;  // optional: the chunk is each sequence's last nq tokens
  int T;
  int32_t *status;
};

struct RowPos {
  long long b;
  int g, i;
};

// row = (b * nq + i) * G + g
__device__ __forceinline__ RowPos row_pos(const RankArgs &a, long long row) {
  RowPos r;
  if (a.rows <= 0x7fffffffLL) {  // 32-bit division where the rows allow it
    const uint32_t r32 = (uint32_t)row, bi = r32 / (uint32_t)a.G;
    r.g = (int)(r32 - bi * (uint32_t)a.G);
    r.i = (int)(bi % (uint32_t)a.nq);
    r.b = (long long)(bi / (uint32_t)a.nq);
  } else {
    r.g = (int)(row % a.G);
    const long long bi = row / a.G;
    r.i = (int)(bi % a.nq);
    r.b = bi / a.nq;
  }
  return r;
}

// One row, by one warp (Smem: WarpListSmem for kListed, else WarpRankSmem).
template <bool kListed, class Smem>
__device__ __forceinline__ void rank_row(const RankArgs &a, long long row, RowPos rp, Smem &sm) {
  const int lane = threadIdx.x & 31;
  const long long b = rp.b;
  const int g = rp.g, i = rp.i;
  int qs = a.q_start;
  if (a.seq_len) {
    const int len = a.seq_len[b];
    if (len < a.nq || len > a.T) {  // an invalid length: an empty set
      for (int s = lane; s < a.S; s += 32) a.idx[row * a.S + s] = -1;
      if (lane == 0 && i == 0 && g == 0) flag_status(a.status, SPARDA_DEV_RANGE);
      return;
    }
    qs = len - a.nq;
  }
  const BlockParts bp = block_parts(qs + i, kBlk, a.n_init, a.n_local);
  const int ncand = bp.cand_hi - bp.cand_lo;
  int32_t *out = a.idx + row * a.S;
  const int nloc = bp.c - bp.local_lo + 1;
  const bool take_all = ncand <= a.k || a.k == 0;
  const int ntop = take_all ? min(ncand, a.k) : a.k;
  // init | top-k | local | -1 padding (the top-k part below unless every
  // candidate, or none, is taken)
  for (int s = lane; s < a.S; s += 32) {
    int v;
    if (s < bp.init_hi) {
      v = s;
    } else if (s < bp.init_hi + ntop) {
      if (!take_all) continue;
      v = bp.cand_lo + (s - bp.init_hi);
    } else if (s < bp.init_hi + ntop + nloc) {
      v = bp.local_lo + (s - bp.init_hi - ntop);
    } else {
      v = -1;
    }
    out[s] = v;
  }
  if (take_all) return;
  const uint32_t *keys = a.keys + ((b * a.G + g) * a.nq + i) * (long long)a.ld + bp.cand_lo;
  uint32_t tau;
  int need;
  int32_t *top = out + bp.init_hi;
  const uint32_t lt = (1u << lane) - 1u;
  if constexpr (kListed) {
    if (ncand >= 1024 && ncand <= kRegKeys * 32) {
      __builtin_assume(ncand >= 1024);  // entries 0..1023 exist: no bound test for them
      // the lane's largest and second-largest keys, all 64 loads in flight at
      // once; the row is not kept in registers: the listing reads it again
      // from L1, and the register search below loads it for the rows the
      // listed threshold does not settle
      uint32_t u1 = 0u, u2 = 0u;
#pragma unroll
      for (int q = 0; q < kRegKeys; ++q) {
        const int e = q * 32 + lane;
        const uint32_t u = e < ncand ? ld_key(keys + e) : 0u;
        u2 = max(u2, min(u1, u));
        u1 = max(u1, u);
      }
      const uint32_t t0 = __reduce_min_sync(0xffffffffu, u2);
      const uint32_t top_key = __reduce_max_sync(0xffffffffu, u1);
      // t0 = 0: a lane with fewer than two keys; t0 = the top key: all listed keys equal
      if (t0 != 0u && t0 < top_key &&
          warp_topk_listed(list_keys_from(keys, ncand, t0, sm), t0, top_key, a.k, sm, top,
                           bp.cand_lo))
        return;
      __syncwarp();
    }
  }
  if (ncand <= kRegKeys * 32) {
    uint32_t kv[kRegKeys];
    uint32_t umin = 0xFFFFFFFFu, umax = 0u;
#pragma unroll
    for (int q = 0; q < kRegKeys; ++q) {
      const int e = q * 32 + lane;
      kv[q] = e < ncand ? ld_key(keys + e) : 0u;
      if (e < ncand) {
        umin = min(umin, kv[q]);
        umax = max(umax, kv[q]);
      }
    }
    umin = __reduce_min_sync(0xffffffffu, umin);
    umax = __reduce_max_sync(0xffffffffu, umax);
    int n_tau;
    // an entry of 0 is empty (a score's key never is), so the search starts at 1
    umin = max(umin, 1u);
    umax = max(umax, umin);
    warp_threshold_reg<kRegKeys>(kv, (uint32_t)ncand, umin, umax, a.k, sm, tau, need,
                                 n_tau);
    if (need == n_tau) {  // every key equal to tau is kept: keep the keys >= tau
      uint32_t n = 0;
#pragma unroll
      for (int q = 0; q < kRegKeys; ++q) {
        const bool keep = kv[q] >= tau;  // tau > 0, so never an empty entry
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        const uint32_t pos = n + __popc(bal & lt);
        if (keep && pos < (uint32_t)a.k) top[pos] = bp.cand_lo + q * 32 + lane;
        n += __popc(bal);
      }
      return;
    }
    // keep keys > tau and the first `need` keys == tau, in block order
    uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
    for (int q = 0; q < kRegKeys; ++q) {
      const uint32_t u = kv[q];
      const bool gt = u > tau, eq = u == tau && u != 0u;
      const uint32_t bgt = __ballot_sync(0xffffffffu, gt), beq = __ballot_sync(0xffffffffu, eq);
      const uint32_t eq_b = n_eq + __popc(beq & lt);
      if (gt || (eq && eq_b < (uint32_t)need)) {
        const uint32_t pos = n_gt + __popc(bgt & lt) + min(eq_b, (uint32_t)need);
        if (pos < (uint32_t)a.k) top[pos] = bp.cand_lo + q * 32 + lane;
      }
      n_gt += __popc(bgt);
      n_eq += __popc(beq);
    }
    return;
  }
  warp_threshold(keys, ncand, a.k, sm, tau, need);
  // keep keys > tau and the first `need` keys == tau, in block order
  uint32_t n_gt = 0, n_eq = 0;
#pragma unroll 2
  for (int base = 0; base < ncand; base += 32) {
    const int e = base + lane;
    const uint32_t u = e < ncand ? ld_key(keys + e) : 0u;
    const bool gt = e < ncand && u > tau, eq = e < ncand && u == tau;
    const uint32_t bgt = __ballot_sync(0xffffffffu, gt), beq = __ballot_sync(0xffffffffu, eq);
    const uint32_t eq_b = n_eq + __popc(beq & lt);
    if (gt || (eq && eq_b < (uint32_t)need)) {
      const uint32_t pos = n_gt + __popc(bgt & lt) + min(eq_b, (uint32_t)need);
      if (pos < (uint32_t)a.k) top[pos] = bp.cand_lo + e;
    }
    n_gt += __popc(bgt);
    n_eq += __popc(beq);
  }
}

// kListed: every row of the chunk has 1024 to 2048 candidates and k <= 64
// (the host checks), and rows try the listed threshold first; rows it does
// not settle, and every row of the other variant, take the binned search on
// the row held in registers (rows of up to 2048 candidates) or in memory.
// One warp per row.
template <bool kListed>
__global__ void __launch_bounds__((kListed ? kRWarpsListed : kRWarps) * 32, kListed ? 4 : 2)
    rank_rows_kernel(RankArgs a) {
  constexpr int kW = kListed ? kRWarpsListed : kRWarps;
  __shared__ std::conditional_t<kListed, WarpListSmem, WarpRankSmem> wsm[kW];
  const int warp = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * kW + warp;
  pdl_trigger();
  pdl_wait();
  if (row < a.rows) rank_row<kListed>(a, row, row_pos(a, row), wsm[warp]);
}

}  // namespace

// Keys per row of the score workspace: the block count rounded up to whole
// tiles (a tile covers kPBlk / pool blocks).
int prefill_ld(int NB, int pool) { return (int)ceil_div_ll(NB, kPBlk / pool) * (kPBlk / pool); }

size_t prefill_select_ws_bytes(const sparda_params &p, int nq, int pool) {
  const int NB = (p.T + kBlk - 1) / kBlk;
  return (((size_t)p.B * p.G * nq * prefill_ld(NB, pool) * 4) + 255) & ~(size_t)255;
}

cudaError_t launch_select_prefill(const sparda_params &p, const uint16_t *F, int nq, int q_start,
                                  const uint16_t *kc, int32_t *idx, void *ws, int32_t *status,
                                  cudaStream_t stream, int pool) {
  if ((long long)p.B * nq * p.G == 0) return cudaSuccess;
  const int NB = (p.T + kBlk - 1) / kBlk;
  const int ld = prefill_ld(NB, pool);
  const int n_rows = pool == 1 ? NB : window_count(p.T);  // key rows per (b, g)
  // F [B][nq][G][d]: dims (d, G, nq, B); Kc [B][G][NB][d]: dims (d, NB, B*G)
  CUtensorMap mF, mK;
  const uint64_t fd[4] = {(uint64_t)kD, (uint64_t)p.G, (uint64_t)nq, (uint64_t)p.B};
  const uint64_t fs[3] = {(uint64_t)kD * 2, (uint64_t)p.G * kD * 2, (uint64_t)nq * p.G * kD * 2};
  const uint32_t fb[4] = {64, 1, kPTok, 1};
  const uint64_t kd[3] = {(uint64_t)kD, (uint64_t)n_rows, (uint64_t)p.B * p.G};
  const uint64_t ks[2] = {(uint64_t)kD * 2, (uint64_t)n_rows * kD * 2};
  const uint32_t kb[3] = {64, kPBlk, 1};
  if (!tc::make_map_nd(&mF, F, 4, fd, fs, fb) || !tc::make_map_nd(&mK, kc, 3, kd, ks, kb))
    return cudaErrorNotSupported;
  auto kern = pool == 1 ? prefill_scores_kernel<1> : prefill_scores_kernel<4>;
  static bool raised[2][64] = {{false}};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!raised[pool == 1 ? 0 : 1][dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem);
    if (e != cudaSuccess) return e;
    raised[pool == 1 ? 0 : 1][dev] = true;
  }
  PScoreArgs sa;
  sa.keys = static_cast<uint32_t *>(ws);
  sa.status = status;
  sa.G = p.G;
  sa.nq = nq;
  sa.NB = NB;
  sa.ld = ld;
  sa.n_rows = n_rows;
  sa.q_start = q_start;
  sa.n_init = p.n_init;
  sa.n_local = p.n_local;
  sa.seq_len = p.seq_len;
  sa.T = p.T;
  const dim3 grid((unsigned)(ld / (kPBlk / pool)), (unsigned)ceil_div_ll(nq, kPTok),
                  (unsigned)(p.B * p.G));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = kPSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mF, mK, sa);
  if (e != cudaSuccess) return e;
  RankArgs ra;
  ra.keys = static_cast<const uint32_t *>(ws);
  ra.idx = idx;
  ra.rows = (long long)p.B * nq * p.G;
  ra.G = p.G;
  ra.nq = nq;
  ra.ld = ld;
  ra.k = p.k;
  ra.n_init = p.n_init;
  ra.n_local = p.n_local;
  ra.q_start = q_start;
  ra.S = p.k + p.n_init + p.n_local;
  ra.seq_len = p.seq_len;
  ra.T = p.T;
  ra.status = status;
  // the listed threshold when every row qualifies: no lengths (the chunk sits
  // at q_start), k <= 64, and 1024 to 2048 candidates from the chunk's first
  // token to its last
  const int nc_first = block_parts(q_start, kBlk, p.n_init, p.n_local).cand_hi - p.n_init;
  const int nc_last = block_parts(q_start + nq - 1, kBlk, p.n_init, p.n_local).cand_hi - p.n_init;
  const bool listed = tuning(p).select_binned == 0 && p.seq_len == nullptr && p.k >= 1 &&
                      p.k <= 64 && nc_first >= 1024 && nc_last <= kRegKeys * 32;
  const int warps = listed ? kRWarpsListed : kRWarps;
  e = launch_pdl(listed ? rank_rows_kernel<true> : rank_rows_kernel<false>,
                 (unsigned)ceil_div_ll(ra.rows, warps), warps * 32, 0, stream, ra);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sparda
