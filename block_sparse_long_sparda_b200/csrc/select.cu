// select.cu -- Forecast block selection: score every candidate block's
// compressed key with the group's Forecast vector(s), keep the k best, and
// join them with the initial and local blocks.  Also the original selector
// in its per-head softmax form (hsm_select_kernel, further down), the
// comparator the Forecast indexer replaces.
//
// Pages cited: [p4 <section>] = the article "SparDA: a fourth projection that
// lets sparse attention prefetch its own KV cache" (ai.thesatyajit.com);
// [p1 <section>] = the SparDA summary page at deepresearch2agi.pages.dev.
//
// [p4 "The fourth projection", Eq. 4]: B_{l+1} = B_init U B_local U
//   f_top(F_l Kc_{l+1}^T, k)
// [p4 "One Forecast head per GQA group"]: one Forecast vector per group, raw
//   dot products, no softmax.  With nf > 1 the kernel is the multi-head
//   baseline selector of the same section (per-head scores summed).
//
// Design (B200): the decode selection is a streaming read of Kc (256 B per
// block per group) with a tiny amount of math, so it is HBM bound.  A problem
// (one query token of one group of one sequence) is split into chunks of up
// to 1024 candidate blocks, as many as fill one wave of two CTAs per SM.  A
// CTA streams its rows into a three-slot shared-memory ring: bulk async
// copies of 128 contiguous rows on the block grid; on the window grid, TMA
// boxes that bring only the three windows inside each of 40 blocks.  Each
// half-warp scores 8 rows per piece: lane l holds dims [8l, 8l+8) of the 8
// rows, multiplies by the Forecast slice, and a butterfly transpose-reduce
// (8 shuffles for 8 rows) leaves the full score of each row in a pair of
// lanes.  Scores become orderable uint32 keys.  The chunks of a problem meet
// through an atomic ticket: the last CTA to finish (no waiting) loads every
// key of the problem from L2 and finds the k-th key exactly -- a register
// sorting network for k <= 64, binned passes otherwise -- and a
// ballot-and-scan pass in block order keeps everything above it plus the
// lowest-index ties, so results come out sorted by block id with ties to the
// lower id, and writes init U top-k U local.  No CTA ever waits for another.
#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"
#include "rank.cuh"
#include "select_dev.cuh"
#include "tc.cuh"

namespace sparda {

namespace {

// Window grid (32-token windows at stride 16, four per 64-token block):
// block j scores as the best of the three windows inside it, 4j, 4j+1 and
// 4j+2; window 4j+3 straddles two blocks and is never read.  A piece is a
// TMA box of kWBlk blocks x those 3 windows x 128 dims, from a 4-D map
// (dims, window in block, block, (b, g)) whose block extent stops at NW / 4,
// where every block's three windows lie inside the tensor; its row r is
// window r % 3 of block r / 3.  The one or two blocks past the map are
// scored with plain loads (score_tail_windows).
constexpr int kWBlk = 40;
constexpr int kWPieceBytes = kWBlk * 3 * kD * 2;  // 30 KB in a 32 KB ring slot

__device__ __forceinline__ void issue_wpiece(const CUtensorMap *map, int blk0, int pc, int pg,
                                             uint8_t *ring, uint64_t *bars) {
  uint64_t *bar = &bars[pc % kRing];
  mbar_arrive_expect_tx(bar, (uint32_t)kWPieceBytes);
  tc::tma_load_4d(ring + (pc % kRing) * kPieceBytes, map, 0, 0, blk0 + pc * kWBlk, pg, bar);
}

// keys[e] for blocks lo + e, e < m; windows at or past wlimit do not exist for
// this sequence and score -inf.  wsc: 128 floats of shared memory.
__device__ bool score_windows(const CUtensorMap *map, const float *fs, int nf, int lo, int m,
                              int wlimit, int pg, uint32_t *keys, float *wsc, uint8_t *ring,
                              uint64_t *bars) {
  const int hw = threadIdx.x >> 4, hl = threadIdx.x & 15;
  const int n_pc = (m + kWBlk - 1) / kWBlk;
  bool ok = true;
#pragma unroll 1
  for (int pc = 0; pc < n_pc; ++pc) {
    const bool landed = mbar_wait_bounded(&bars[pc % kRing], (uint32_t)((pc / kRing) & 1));
    if (__syncthreads_or(!landed)) {
      ok = false;
      if (threadIdx.x == 0)
        for (int q = pc; q < min(n_pc, pc + kRing); ++q)
          (void)mbar_wait_bounded(&bars[q % kRing], (uint32_t)((q / kRing) & 1));
      __syncthreads();
      break;
    }
    const int nblk = min(kWBlk, m - pc * kWBlk);
    const int rows = 3 * nblk;
    const uint8_t *piece = ring + (pc % kRing) * kPieceBytes;
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
    const int r = row0 + (hl >> 1);  // 0..127
    if ((hl & 1) == 0) {
      const int w = 4 * (lo + pc * kWBlk + r / 3) + r % 3;  // its window
      wsc[r] = (r < rows && w < wlimit) ? sc : -INFINITY;
    }
    __syncthreads();
    if ((int)threadIdx.x < nblk) {
      const int t = threadIdx.x;
      keys[pc * kWBlk + t] = orderable_key(fmaxf(fmaxf(wsc[3 * t], wsc[3 * t + 1]), wsc[3 * t + 2]));
    }
    __syncthreads();  // piece and row scores consumed
    if (threadIdx.x == 0 && pc + kRing < n_pc) issue_wpiece(map, lo, pc + kRing, pg, ring, bars);
  }
  return ok;
}

// keys[e] for blocks lo + e, m <= e < n (past the map's block extent, at most
// two): one warp per (block, window), plain loads of the window's key row.
__device__ void score_tail_windows(const uint16_t *kw_bg, const float *fs, int nf, int lo, int m,
                                   int n, int wlimit, uint32_t *keys, float *wsc) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int items = (n - m) * 3;
  for (int it = warp; it < items; it += kSelThreads / 32) {
    const int w = 4 * (lo + m + it / 3) + it % 3;
    float s = -INFINITY;
    if (w < wlimit) {  // uniform over the warp
      const uint2 kv = *reinterpret_cast<const uint2 *>(kw_bg + (long long)w * kD + lane * 4);
      float acc = 0.f;
      for (int f = 0; f < nf; ++f) {
        const float4 q = *reinterpret_cast<const float4 *>(fs + f * kD + lane * 4);
        acc += q.x * bf16_lo(kv.x) + q.y * bf16_hi(kv.x) + q.z * bf16_lo(kv.y) + q.w * bf16_hi(kv.y);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      s = acc;
    }
    if (lane == 0) wsc[it] = s;
  }
  __syncthreads();
  for (int e = m + (int)threadIdx.x; e < n; e += kSelThreads) {
    const int t = e - m;
    keys[e] = orderable_key(fmaxf(fmaxf(wsc[3 * t], wsc[3 * t + 1]), wsc[3 * t + 2]));
  }
  __syncthreads();
}

template <int kPool, bool kCached = false>
__global__ void __launch_bounds__(kSelThreads, 2)
    select_kernel(const __grid_constant__ CUtensorMap mapW, SelArgs a) {
  // dynamic shared memory, the ring aligned to 128 bytes by hand (a TMA
  // destination): piece ring | scoring vectors (fp32) | score keys
  extern __shared__ __align__(128) uint8_t dyn_raw[];
  uint8_t *ring = dyn_raw + ((128u - (smem_addr(dyn_raw) & 127u)) & 127u);
  float *fs = reinterpret_cast<float *>(ring + kRing * kPieceBytes);
  uint32_t *dyn = reinterpret_cast<uint32_t *>(ring + kRing * kPieceBytes + a.nf * kD * 4);
  __shared__ __align__(8) uint64_t bars[kRing];
  __shared__ RankSmem rs;
  __shared__ float wsc[128];  // window grid: row scores of a piece
  __shared__ int s_last, s_failed;

  pdl_trigger();
  pdl_wait();
  if constexpr (kPool == 1) {  // the block grid (select_dev.cuh), optionally with the slot cache
    __shared__ int s_flags[2];
    SelSmem sm;
    sm.ring = ring;
    sm.fs = fs;
    sm.keys = dyn;
    sm.rank_keys = dyn;
    sm.scratch = reinterpret_cast<uint32_t *>(ring);
    sm.bars = bars;
    sm.rs = &rs;
    sm.flags = s_flags;
    select_block_item<kRing, kCached>(a, blockIdx.x, sm);
    return;
  }
  // problems are laid out chunk-fastest so a problem's chunks run together
  // and its merge overlaps the streaming of later problems
  const long long prob = blockIdx.x / a.n_chunks;
  const int chunk = (int)(blockIdx.x - prob * a.n_chunks);
  const int g = (int)(prob % a.G);
  const long long bi = prob / a.G;
  const int i = (int)(bi % a.nq);
  const long long b = bi / a.nq;
  int pos = a.q_start + i;
  int32_t *out = a.idx + prob * a.S;
  int rows_b = a.NB;  // key rows of this sequence (the row stride stays a.NB)
  if (a.seq_len) {  // per-sequence lengths: the queries are the sequence's last nq tokens
    const int len = a.seq_len[b];
    if (len < a.nq || len > a.T) {  // an invalid length: an empty set
      if (chunk == 0) {
        for (int s2 = threadIdx.x; s2 < a.S; s2 += kSelThreads) out[s2] = -1;
        if (threadIdx.x == 0) flag_status(a.status, SPARDA_DEV_RANGE);
      }
      if (a.n_chunks > 1) {  // keep the ticket count of the problem right
        __syncthreads();
        if (threadIdx.x == 0) {
          const unsigned t = atomicAdd(&a.counters[prob], 1u);
          if (t == (unsigned)(a.n_chunks - 1)) a.counters[prob] = 0u;
        }
      }
      return;
    }
    pos = len - a.nq + i;
    if (kPool > 1) rows_b = window_count(len);
  }
  const BlockParts bp = block_parts(pos, kBlk, a.n_init, a.n_local);
  const int ncand = bp.cand_hi - bp.cand_lo;

  if (ncand <= a.k || a.k == 0) {  // nothing to rank: every candidate, or none, is kept
    if (chunk == 0) write_set(out, bp, min(ncand, a.k), a.S, true);
    return;
  }

  uint32_t *keys = dyn;
  const int lo = bp.cand_lo + chunk * a.CH;
  const int n = max(0, min(bp.cand_hi, lo + a.CH) - lo);
  // key rows of this chunk: blocks, or (window grid) 4 windows per block, the
  // last ones clipped to the windows that exist
  const int row_lo = lo * kPool;
  const int n_rows = kPool == 1 ? n : max(0, min(n * kPool, rows_b - row_lo));
  const int pg = (int)(b * a.G + g);  // (sequence, group): the key tensor's problem index
  const uint16_t *kc_bg = a.kc + (long long)pg * a.NB * kD;
  // window grid: blocks [lo, lo + m) come by TMA, the rest by plain loads
  const int m = kPool == 1 ? 0 : max(0, min(lo + n, a.NBf) - lo);
  if (threadIdx.x == 0) {
    for (int q = 0; q < kRing; ++q) mbar_init(&bars[q], 1);
    fence_mbar_init();
    if (kPool == 1) {
      prime_ring(kc_bg, row_lo, n_rows, ring, bars);
    } else if (m > 0) {  // the map exists whenever a block comes by TMA
      tc::prefetch_map(&mapW);
      for (int pc = 0; pc < min(kRing, (m + kWBlk - 1) / kWBlk); ++pc)
        issue_wpiece(&mapW, lo, pc, pg, ring, bars);
    }
  }
  // Forecast vector(s) of this problem -> fp32 in shared memory
  const uint16_t *f = a.F + (bi * a.G + g) * (long long)a.nf * kD;
  for (int t = threadIdx.x; t < a.nf * kD; t += kSelThreads)
    fs[t] = __uint_as_float(((uint32_t)f[t]) << 16);
  __syncthreads();

  if (kPool > 1) {  // blocks whose windows all lie past the clipped rows keep a valid key
    for (int e = threadIdx.x; e < n; e += kSelThreads) keys[e] = orderable_key(-INFINITY);
    __syncthreads();
  }
  bool ok;
  if (kPool == 1) {
    ok = score_rows(kc_bg, fs, a.nf, row_lo, n_rows, keys, ring, bars);
  } else {
    ok = score_windows(&mapW, fs, a.nf, lo, m, row_lo + n_rows, pg, keys, wsc, ring, bars);
    if (ok && m < n) score_tail_windows(kc_bg, fs, a.nf, lo, m, n, row_lo + n_rows, keys, wsc);
  }
  // a copy that never landed: the problem's set is reported empty rather
  // than wrong (by the last chunk, when there are several)
  if (!ok && threadIdx.x == 0) flag_status(a.status, SPARDA_DEV_TIMEOUT);
  __syncthreads();

  uint32_t tau = 0;
  int need = 0;
  int32_t *top = out + bp.init_hi;

  if (a.n_chunks == 1) {  // n == ncand > k: rank in shared memory
    if (!ok) {
      for (int s2 = threadIdx.x; s2 < a.S; s2 += kSelThreads) out[s2] = -1;
      return;
    }
    if (a.k <= kTopkMaxK && n <= kTopkMaxN && !a.old_rank)
      find_threshold_topk(keys, n, a.k, reinterpret_cast<uint32_t *>(ring), rs, tau, need);
    else
      find_threshold(keys, n, a.k, rs, tau, need);
    const int ntop = compact_kept(keys, n, tau, need, a.k, rs,
                                  [&](int pos, int e) { st_list(top + pos, bp.cand_lo + e); });
    write_set(out, bp, ntop, a.S, false);
    return;
  }

  // ---- chunk scores -> workspace; the last chunk to finish ranks them all.
  // A chunk whose copy never landed still takes its ticket (so the count
  // completes and the last chunk resets it) and raises the problem's flag ----
  uint32_t *pkeys = a.cand_key + prob * (long long)a.cap;
  if (ok)
    for (int e = threadIdx.x; e < n; e += kSelThreads) pkeys[chunk * a.CH + e] = keys[e];
  else if (threadIdx.x == 0)
    a.failed[prob] = 1u;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned t = atomicAdd(&a.counters[prob], 1u);
    s_last = (t == (unsigned)(a.n_chunks - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x == 0) s_failed = (int)__ldcg(a.failed + prob);
  __syncthreads();
  if (s_failed) {
    for (int s2 = threadIdx.x; s2 < a.S; s2 += kSelThreads) out[s2] = -1;
    if (threadIdx.x == 0) {
      a.failed[prob] = 0u;
      a.counters[prob] = 0u;
    }
    return;
  }
  for (int e = threadIdx.x; e < ncand; e += kSelThreads) keys[e] = __ldcg(pkeys + e);
  __syncthreads();
  if (a.k <= kTopkMaxK && ncand <= kTopkMaxN && !a.old_rank)
    find_threshold_topk(keys, ncand, a.k, reinterpret_cast<uint32_t *>(ring), rs, tau, need);
  else
    find_threshold(keys, ncand, a.k, rs, tau, need);
  const int ntop = compact_kept(keys, ncand, tau, need, a.k, rs,
                                [&](int pos, int e) { st_list(top + pos, bp.cand_lo + e); });
  write_set(out, bp, ntop, a.S, false);
  if (threadIdx.x == 0) a.counters[prob] = 0u;
}

// ---------------------------------------------------------------------------
// the original selector in its per-head softmax form: for every query head h
// of the group, a softmax over all key rows the query sees of q_h . k_r / tau,
// summed over the heads; on the window grid a block weighs as much as its
// heaviest window.  ["SparDA: a fourth projection..." article, "Training:
// distilling the selector you already have", Eq. 6; "One Forecast head per
// GQA group": the baseline scores with every query head.]
//
// The softmax needs each head's max and normaliser over every seen row --
// the initial and local rows and the straddling windows too, which are never
// ranked -- so the chunks of a problem cover all seen rows, not only the
// candidates.  A chunk streams its rows once, writes each head's scores to
// the workspace and keeps a running (max, sum of exp(s - max)) per head; the
// last chunk to finish merges those into (M_h, Z_h), turns the candidates'
// scores into weights sum_h exp(s_h - M_h) / Z_h, and ranks them exactly as
// select_kernel ranks raw scores (same threshold search and compaction, so
// the same tie rule).
// ---------------------------------------------------------------------------
constexpr int kHsmMaxHeads = 16;

struct HsmArgs {
  const int32_t *seq_len;
  int32_t *status;     // optional device status word
  const uint16_t *Q;   // [B][G][nf][d]; the keys [B][G][NR][d] come through a tensor map
  int32_t *idx;        // [B][G][S]
  uint32_t *counters;  // [problem] tickets
  uint32_t *failed;    // [problem] set when a chunk's copy never landed
  float2 *stats;       // [problem][n_chunks][nf] (max, sum of exp(s - max))
  float *scores;       // [problem][nf][rows_cap] q_h . k_r / tau
  int G, nf, NR, k, n_init, n_local, q_start, S, T;
  int CH, n_chunks, rows_cap;  // CH blocks per chunk
  float inv_tau;
  int old_rank;
};

// (m, z) pairs of two row sets -> the pair of their union
__device__ __forceinline__ void merge_stat(float &m, float &z, float mo, float zo) {
  const float mm = fmaxf(m, mo);
  z = mm == -INFINITY ? 0.f : z * expf(m - mm) + zo * expf(mo - mm);
  m = mm;
}

// the group's heads as the MMA's B operand: [2 dim halves][16 heads][64 dims]
constexpr int kHsmOpB = 2 * 16 * 128;
constexpr int kHsmTmemCols = 32;  // two 16-column score stages

// one 128-row piece of key rows by TMA (two 64-dim halves, 128-byte swizzle)
__device__ __forceinline__ void hsm_issue_piece(const CUtensorMap *map, int row_lo, int pc,
                                                int prob, uint8_t *ring, uint64_t *bars) {
  uint64_t *bar = &bars[pc % kRing];
  uint8_t *dst = ring + (pc % kRing) * kPieceBytes;
  mbar_arrive_expect_tx(bar, (uint32_t)kPieceBytes);
  const int y = row_lo + pc * kPieceRows;
  tc::tma_load_3d(dst, map, 0, y, prob, bar);
  tc::tma_load_3d(dst + kPieceBytes / 2, map, 64, y, prob, bar);
}

template <int kPool, int NFT>
__global__ void __launch_bounds__(kSelThreads, 2)
    hsm_select_kernel(const __grid_constant__ CUtensorMap mapKc, HsmArgs a) {
  // dynamic shared memory, aligned to 1024 bytes by hand (the swizzle atom):
  // piece ring | head operand | weight keys
  extern __shared__ __align__(128) uint8_t hsm_dyn[];
  uint8_t *ring = hsm_dyn + ((1024u - (smem_addr(hsm_dyn) & 1023u)) & 1023u);
  uint8_t *opB = ring + kRing * kPieceBytes;
  uint32_t *keys = reinterpret_cast<uint32_t *>(opB + kHsmOpB);
  __shared__ __align__(8) uint64_t bars[kRing + 2];  // piece landed x kRing, MMA done x 2 stages
  __shared__ uint32_t tmem_slot;
  __shared__ RankSmem rs;
  __shared__ float2 wstat[kSelThreads / 32][kHsmMaxHeads];
  __shared__ float s_m[kHsmMaxHeads], s_iz[kHsmMaxHeads];
  __shared__ int s_last, s_failed;

  pdl_trigger();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long prob = blockIdx.x / a.n_chunks;  // = b * G + g
  const int chunk = (int)(blockIdx.x - prob * a.n_chunks);
  const long long b = prob / a.G;
  int pos = a.q_start;
  int32_t *out = a.idx + prob * a.S;
  if (a.seq_len) {  // the query is the sequence's last token
    const int len = a.seq_len[b];
    if (len < 1 || len > a.T) {  // an invalid length: an empty set (every chunk returns here)
      if (chunk == 0) {
        for (int s2 = tid; s2 < a.S; s2 += kSelThreads) out[s2] = -1;
        if (tid == 0) flag_status(a.status, SPARDA_DEV_RANGE);
      }
      return;
    }
    pos = len - 1;
  }
  const BlockParts bp = block_parts(pos, kBlk, a.n_init, a.n_local);
  const int ncand = bp.cand_hi - bp.cand_lo;
  if (ncand <= a.k || a.k == 0) {  // nothing to rank (every chunk returns here)
    if (chunk == 0) write_set(out, bp, min(ncand, a.k), a.S, true);
    return;
  }

  // the rows the query sees: blocks 0..c, or the windows complete by pos
  const int dom_blocks = bp.c + 1;
  const int dom_rows = kPool == 1 ? min(dom_blocks, a.NR) : min(window_count(pos + 1), a.NR);
  const int blo = chunk * a.CH;
  const int row_lo = blo * kPool;
  const int n_rows = max(0, min(min(dom_blocks, blo + a.CH) * kPool, dom_rows) - row_lo);
  const int n_pc = (n_rows + kPieceRows - 1) / kPieceRows;
  float m_run[NFT], z_run[NFT];
#pragma unroll
  for (int f = 0; f < NFT; ++f) {
    m_run[f] = -INFINITY;
    z_run[f] = 0.f;
  }
  float *sc = a.scores + prob * (long long)a.nf * a.rows_cap;
  bool ok = true;

  // ---- scores of the chunk's rows on the tensor cores: for each 128-row
  // piece, D[row][head] = Kc_piece . Q^T (M = 128 rows, N = 16 heads, K = 128
  // in eight steps), D double-buffered in TMEM so the product of the next
  // piece runs while warps 0-3 read this one (thread = row = TMEM lane) ----
  if (n_pc > 0) {
    if ((smem_addr(ring) & 1023u) != 0u) {  // cannot happen with the sizes launched
      ok = false;
      if (tid == 0) flag_status(a.status, SPARDA_DEV_LAYOUT);
    } else {
      if (tid == 0) {
        for (int q = 0; q < kRing + 2; ++q) mbar_init(&bars[q], 1);
        fence_mbar_init();
        tc::prefetch_map(&mapKc);
        for (int pc = 0; pc < min(kRing, n_pc); ++pc)
          hsm_issue_piece(&mapKc, row_lo, pc, (int)prob, ring, bars);
      }
      {  // heads -> B operand (rows >= nf are zero); 256 threads, one 16-byte chunk each
        const int half = tid >> 7, row = (tid >> 3) & 15, ch = tid & 7;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (row < a.nf)
          v = *reinterpret_cast<const uint4 *>(a.Q + (prob * a.nf + row) * (long long)kD + half * 64 + ch * 8);
        *reinterpret_cast<uint4 *>(opB + half * (kHsmOpB / 2) + tc::sw128_offset(row, ch * 8)) = v;
        fence_proxy_async_smem();
      }
      if (warp == 0) tc::tmem_alloc(&tmem_slot, kHsmTmemCols);
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      const uint32_t tmem = tmem_slot;
      constexpr uint32_t idesc = tc::idesc_bf16(kPieceRows, 16, false, false);
      int n_issued = 0, n_loaded = min(kRing, n_pc);  // thread 0's view
      auto issue_mma = [&](int pc) -> bool {  // thread 0
        if (!mbar_wait_bounded(&bars[pc % kRing], (uint32_t)((pc / kRing) & 1))) return false;
        tc::fence_after_sync();
        const uint8_t *pa = ring + (pc % kRing) * kPieceBytes;
        const uint32_t d = tmem + (uint32_t)((pc & 1) * 16);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_bf16(d, tc::sdesc(pa + (kk >> 2) * (kPieceBytes / 2) + (kk & 3) * 32, 16, 1024),
                       tc::sdesc(opB + (kk >> 2) * (kHsmOpB / 2) + (kk & 3) * 32, 16, 1024), idesc,
                       kk > 0);
        tc::mma_commit(&bars[kRing + (pc & 1)]);
        n_issued = pc + 1;
        return true;
      };
      int bad = 0;
      if (tid == 0) bad = !issue_mma(0);
      bad = __syncthreads_or(bad);
      int pc = 0;
#pragma unroll 1
      for (; !bad && pc < n_pc; ++pc) {
        int fail = 0;
        if (tid == 0 && pc + 1 < n_pc) fail = !issue_mma(pc + 1);
        if (warp < 4) {
          const bool done = mbar_wait_bounded(&bars[kRing + (pc & 1)], (uint32_t)((pc >> 1) & 1));
          if (__all_sync(0xffffffffu, done)) {
            tc::fence_after_sync();
            float v[16];
            tc::tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)((pc & 1) * 16), v);
            const int rows = min(kPieceRows, n_rows - pc * kPieceRows);
            if (tid < rows) {
              const long long grow = (long long)row_lo + pc * kPieceRows + tid;
#pragma unroll
              for (int f = 0; f < NFT; ++f) {
                if (f < a.nf) {
                  const float s = v[f] * a.inv_tau;
                  sc[(long long)f * a.rows_cap + grow] = s;
                  if (s > m_run[f]) {
                    z_run[f] = z_run[f] * expf(m_run[f] - s) + 1.f;
                    m_run[f] = s;
                  } else {
                    z_run[f] += expf(s - m_run[f]);
                  }
                }
              }
            }
          } else {
            fail = 1;
          }
        }
        tc::fence_before_sync();
        bad = __syncthreads_or(fail);
        // piece pc's product is done: its ring slot takes piece pc + kRing
        if (!bad && tid == 0 && pc + kRing < n_pc) {
          hsm_issue_piece(&mapKc, row_lo, pc + kRing, (int)prob, ring, bars);
          n_loaded = pc + kRing + 1;
        }
      }
      if (bad) {
        ok = false;
        if (tid == 0) {  // let copies and products in flight finish (bounded) before release
          flag_status(a.status, SPARDA_DEV_TIMEOUT);
          for (int q = pc; q < n_loaded; ++q)
            (void)mbar_wait_bounded(&bars[q % kRing], (uint32_t)((q / kRing) & 1));
          if (n_issued > 0)
            (void)mbar_wait_bounded(&bars[kRing + ((n_issued - 1) & 1)],
                                    (uint32_t)(((n_issued - 1) >> 1) & 1));
        }
      }
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      if (warp == 0) tc::tmem_dealloc(tmem, kHsmTmemCols);
    }
  }
  if (!ok && tid == 0) a.failed[prob] = 1u;

  // this chunk's (max, normaliser) per head
#pragma unroll
  for (int f = 0; f < NFT; ++f) {
    if (f < a.nf) {
      float m = m_run[f], z = z_run[f];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o);
        const float zo = __shfl_xor_sync(0xffffffffu, z, o);
        merge_stat(m, z, mo, zo);
      }
      if (lane == 0) wstat[warp][f] = make_float2(m, z);
    }
  }
  __syncthreads();
  if (tid < a.nf) {
    float m = wstat[0][tid].x, z = wstat[0][tid].y;
    for (int w = 1; w < kSelThreads / 32; ++w) merge_stat(m, z, wstat[w][tid].x, wstat[w][tid].y);
    a.stats[(prob * a.n_chunks + chunk) * a.nf + tid] = make_float2(m, z);
  }

  // ---- the last chunk to finish weighs and ranks the candidates ----
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicAdd(&a.counters[prob], 1u);
    s_last = (t == (unsigned)(a.n_chunks - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid == 0) s_failed = (int)__ldcg(a.failed + prob);
  if (tid < a.nf) {
    float M = -INFINITY, Z = 0.f;
    for (int ch = 0; ch < a.n_chunks; ++ch) {
      const float2 st = __ldcg(a.stats + (prob * a.n_chunks + ch) * a.nf + tid);
      merge_stat(M, Z, st.x, st.y);
    }
    s_m[tid] = Z > 0.f ? M : 0.f;
    s_iz[tid] = Z > 0.f ? 1.f / Z : 0.f;
  }
  __syncthreads();
  if (s_failed) {  // a copy never landed: report an empty set rather than a wrong one
    for (int s2 = tid; s2 < a.S; s2 += kSelThreads) out[s2] = -1;
    if (tid == 0) {
      a.failed[prob] = 0u;
      a.counters[prob] = 0u;
    }
    return;
  }
  // Weights of the candidates as keys.  A thread takes 8 candidates at a
  // time and, head by head, issues all their loads before using any, so the
  // L2 latency is paid once per head, not once per value; on the window grid
  // one 16-byte load brings a block's four windows (the fourth, straddling
  // one is not pooled).
  constexpr int kW = kPool == 1 ? 1 : 3;
#pragma unroll 1
  for (int base = 0; base < ncand; base += 8 * kSelThreads) {
    float x[8][kW];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int rr = 0; rr < kW; ++rr) x[i][rr] = 0.f;
#pragma unroll 1
    for (int f = 0; f < a.nf; ++f) {
      const float *scf = sc + (long long)f * a.rows_cap;
      float v[8][kW];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = base + i * kSelThreads + tid;
        const int j = bp.cand_lo + min(e, ncand - 1);  // past the end: a valid row, unused
        if (kPool == 1) {
          v[i][0] = __ldcg(scf + j);
        } else {
          const float4 q4 = __ldcg(reinterpret_cast<const float4 *>(scf + 4LL * j));
          v[i][0] = q4.x;
          v[i][kW > 1 ? 1 : 0] = q4.y;
          v[i][kW > 2 ? 2 : 0] = q4.z;
        }
      }
      const float mf = s_m[f], izf = s_iz[f];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int rr = 0; rr < kW; ++rr) x[i][rr] += expf(v[i][rr] - mf) * izf;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = base + i * kSelThreads + tid;
      if (e < ncand) {
        const int j = bp.cand_lo + e;
        float w = -INFINITY;
#pragma unroll
        for (int rr = 0; rr < kW; ++rr)
          if (j * kPool + rr < dom_rows) w = fmaxf(w, x[i][rr]);  // windows that exist
        keys[e] = orderable_key(w);
      }
    }
  }
  __syncthreads();
  uint32_t tau = 0;
  int need = 0;
  if (a.k <= kTopkMaxK && ncand <= kTopkMaxN && !a.old_rank)
    find_threshold_topk(keys, ncand, a.k, reinterpret_cast<uint32_t *>(ring), rs, tau, need);
  else
    find_threshold(keys, ncand, a.k, rs, tau, need);
  int32_t *top = out + bp.init_hi;
  const int ntop = compact_kept(keys, ncand, tau, need, a.k, rs,
                                [&](int p2, int e) { st_list(top + p2, bp.cand_lo + e); });
  write_set(out, bp, ntop, a.S, false);
  if (tid == 0) a.counters[prob] = 0u;
}

}  // namespace

// The plan depends on the shapes only (not on where the query chunk sits), so
// the workspace size is known before the call: chunking is sized for a query
// at the end of the sequence, the most candidates any query can have.
SelectPlan plan_select(const sparda_params &p, int nq, int nf, int pool) {
  SelectPlan pl{};
  pl.n_problems = (long long)p.B * nq * p.G;
  const BlockParts bp = block_parts(p.T - 1, kBlk, p.n_init, p.n_local);
  pl.ncand_max = bp.cand_hi - bp.cand_lo;
  pl.CH = kSelThreads;
  pl.n_chunks = 1;
  pl.kc = 0;
  pl.tensor_scores = 0;
  pl.ws_bytes = 0;
  if (pl.ncand_max <= p.k || p.k == 0 || pl.n_problems == 0) return pl;
  if (nf == 1 && nq >= kPrefillTensorMinQ && tuning(p).select_stream == 0) {
    // a chunk of query tokens: the scores are a dense product per (sequence,
    // group), computed on the tensor cores and kept in the workspace
    pl.tensor_scores = 1;
    pl.ws_bytes = prefill_select_ws_bytes(p, nq, pool);
    return pl;
  }

  const int forced = tuning(p).select_chunk;
  int CH;
  if (forced > 0) {
    CH = std::max(kSelThreads, (forced / kSelThreads) * kSelThreads);
  } else {
    // as many chunks per problem as fill one wave of resident CTAs (two per
    // SM), at least 256 candidates each: the streams of one wave overlap
    // best, and every later wave would restart them; one chunk per problem
    // once there are plenty of problems (prefill)
    static int sm_count[64] = {0};  // per device, queried once
    int dev = 0, n_sm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
      if (sm_count[dev] == 0 &&
          cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sm_count[dev] = 148;
      n_sm = sm_count[dev];
    }
    (void)cudaGetLastError();
    const long long wave = 2LL * n_sm;
    const long long per = std::max<long long>(1, wave / std::max<long long>(1, pl.n_problems));
    CH = (int)(ceil_div_ll(ceil_div_ll(pl.ncand_max, per), kSelThreads) * kSelThreads);
    // longer streams per CTA stop paying past 1024 blocks, on both grids
    // (the window grid reads three windows per block): one wave of
    // 1024-block chunks beat 256- and 512-block ones at B = 16, T = 128K,
    // with one length for all and with the real models' mixed lengths
    CH = std::min(std::max(CH, kSelThreads), 1024);
    if (pl.n_problems >= 8LL * n_sm) CH = kMaxCand;
  }
  if (CH >= pl.ncand_max) CH = std::min(kMaxCand, (int)ceil_div_ll(pl.ncand_max, kSelThreads) * kSelThreads);
  pl.CH = CH;
  pl.n_chunks = (int)ceil_div_ll(pl.ncand_max, CH);
  if (pl.n_chunks > 1) {
    pl.kc = pl.ncand_max;  // every candidate's key is kept for the final rank
    size_t off = 2 * (((size_t)pl.n_problems * 4 + 255) & ~(size_t)255);  // tickets, flags
    off += (((size_t)pl.n_problems * pl.n_chunks * CH * 4) + 255) & ~(size_t)255;  // keys
    pl.ws_bytes = off;
  }
  return pl;
}

int select_supported(const SelectPlan &pl) {
  if (pl.tensor_scores) return 1;
  if (pl.CH > kMaxCand) return 0;
  if (pl.ncand_max > kMaxCand) return 0;
  return 1;
}

cudaError_t launch_select(const sparda_params &p, const SelectPlan &pl, const uint16_t *F, int nq,
                          int nf, int q_start, const uint16_t *kc, int32_t *idx, void *ws,
                          int32_t *status, cudaStream_t stream, int pool, const SelCache *cache) {
  if (pl.n_problems == 0) return cudaSuccess;
  if (pl.tensor_scores)
    return launch_select_prefill(p, F, nq, q_start, kc, idx, ws, status, stream, pool);
  SelArgs a;
  a.status = status;
  a.failed = nullptr;
  a.seq_len = p.seq_len;
  a.T = p.T;
  a.F = F;
  a.kc = kc;
  a.idx = idx;
  a.nq = nq;
  a.G = p.G;
  a.nf = nf;
  a.NB = pool == 1 ? (p.T + kBlk - 1) / kBlk : window_count(p.T);  // key rows per (b, g)
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
  a.old_rank = tuning(p).select_binned != 0 ? 1 : 0;
  a.cc = SelCache{};
  if (cache) {  // decode on the block grid only, with the step's words inside the ring
    if (pool != 1 || nq != 1 || cache->C < a.S ||
        cache_step_words(cache->C, a.S) * 4 > (long long)kRing * kPieceBytes)
      return cudaErrorNotSupported;
    a.cc = *cache;
  }
  // window grid: key rows [B*G][NW][d] as (dims, window in block, block, (b, g)),
  // three of every four windows, blocks up to NW / 4 (all three windows inside)
  CUtensorMap mW{};
  a.NBf = 0;
  if (pool != 1) {
    a.NBf = a.NB / 4;
    if (a.NBf > 0) {
      const uint64_t wdim[4] = {(uint64_t)kD, 3, (uint64_t)a.NBf, (uint64_t)p.B * p.G};
      const uint64_t wstr[3] = {(uint64_t)kD * 2, (uint64_t)4 * kD * 2, (uint64_t)a.NB * kD * 2};
      const uint32_t wbox[4] = {(uint32_t)kD, 3, (uint32_t)kWBlk, 1};
      if (!tc::make_map_nd(&mW, kc, 4, wdim, wstr, wbox, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorNotSupported;
    }
  }
  size_t smem = 128 + (size_t)kRing * kPieceBytes + (size_t)nf * kD * 4 + (size_t)pl.CH * 4;
  if (pl.n_chunks > 1) {
    char *w = static_cast<char *>(ws);
    const size_t words = ((size_t)pl.n_problems * 4 + 255) & ~(size_t)255;
    a.counters = reinterpret_cast<uint32_t *>(w);
    a.failed = reinterpret_cast<uint32_t *>(w + words);
    a.cand_key = reinterpret_cast<uint32_t *>(w + 2 * words);
    smem = 128 + (size_t)kRing * kPieceBytes + (size_t)nf * kD * 4 +
           (size_t)std::max(pl.CH, pl.ncand_max) * 4;
  }
  auto kern = cache ? select_kernel<1, true> : pool == 1 ? select_kernel<1> : select_kernel<4>;
  {  // raised once per device and kernel to the largest size used; most
     // shared memory goes to the ring, so prefer the largest carveout
    static size_t raised[3][64] = {{0}};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    size_t &r = raised[cache ? 2 : pool == 1 ? 0 : 1][dev];
    if (r < smem) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e != cudaSuccess) return e;
      r = smem;
    }
  }
  const long long grid = pl.n_problems * pl.n_chunks;
  const cudaError_t e = launch_pdl(kern, (unsigned)grid, kSelThreads, smem, stream, mW, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Chunks cover the seen blocks 0..c of a query at the end of the sequence
// (the most any query has), sized by the same one-wave rule as plan_select.
HsmPlan plan_head_softmax(const sparda_params &p, int nf, int pool) {
  HsmPlan pl{};
  pl.n_problems = (long long)p.B * p.G;
  const BlockParts bp = block_parts(p.T - 1, kBlk, p.n_init, p.n_local);
  pl.ncand_max = bp.cand_hi - bp.cand_lo;
  const int dom = bp.c + 1;
  pl.CH = dom;
  pl.n_chunks = 1;
  pl.rows_cap = 0;
  pl.ws_bytes = 0;
  if (pl.ncand_max <= p.k || p.k == 0 || pl.n_problems == 0) return pl;
  const int forced = tuning(p).select_chunk;
  int CH;
  if (forced > 0) {
    CH = std::max(kSelThreads, (forced / kSelThreads) * kSelThreads);
  } else {
    static int sm_count[64] = {0};
    int dev = 0, n_sm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
      if (sm_count[dev] == 0 &&
          cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sm_count[dev] = 148;
      n_sm = sm_count[dev];
    }
    (void)cudaGetLastError();
    const long long wave = 2LL * n_sm;
    const long long per = std::max<long long>(1, wave / pl.n_problems);
    CH = (int)(ceil_div_ll(ceil_div_ll(dom, per), kSelThreads) * kSelThreads);
    // on both grids chunks of up to 1024 blocks: with the scores on the
    // tensor cores a chunk streams 1 MB of window keys as fast as 256 KB of
    // block keys, and one wave of long streams beat four waves of short ones
    // (75.7 -> 63.4 us on window keys at B = 16, T = 128K)
    CH = std::min(std::max(CH, kSelThreads), 1024);
  }
  pl.CH = std::min(CH, (int)ceil_div_ll(dom, kSelThreads) * kSelThreads);
  pl.n_chunks = (int)ceil_div_ll(dom, pl.CH);
  pl.rows_cap = pl.n_chunks * pl.CH * pool;
  size_t off = 2 * (((size_t)pl.n_problems * 4 + 255) & ~(size_t)255);  // tickets, failure flags
  off += ((size_t)pl.n_problems * pl.n_chunks * nf * 8 + 255) & ~(size_t)255;  // chunk stats
  off += (size_t)pl.n_problems * nf * pl.rows_cap * 4;                      // head scores
  pl.ws_bytes = off;
  return pl;
}

int head_softmax_supported(const HsmPlan &pl, int nf) {
  if (nf < 1 || nf > kHsmMaxHeads) return 0;
  if (pl.ncand_max > kMaxCand) return 0;
  return 1;
}

cudaError_t launch_head_softmax(const sparda_params &p, const HsmPlan &pl, const uint16_t *Q,
                                int nf, int q_start, float tau, const uint16_t *kc, int32_t *idx,
                                void *ws, int32_t *status, cudaStream_t stream, int pool) {
  if (pl.n_problems == 0) return cudaSuccess;
  HsmArgs a;
  a.seq_len = p.seq_len;
  a.status = status;
  a.Q = Q;
  a.idx = idx;
  a.G = p.G;
  a.nf = nf;
  a.NR = pool == 1 ? (p.T + kBlk - 1) / kBlk : window_count(p.T);
  a.k = p.k;
  a.n_init = p.n_init;
  a.n_local = p.n_local;
  a.q_start = q_start;
  a.S = p.k + p.n_init + p.n_local;
  a.T = p.T;
  a.CH = pl.CH;
  a.n_chunks = pl.n_chunks;
  a.rows_cap = pl.rows_cap;
  a.inv_tau = 1.f / tau;
  a.old_rank = tuning(p).select_binned != 0 ? 1 : 0;
  a.counters = nullptr;
  a.failed = nullptr;
  a.stats = nullptr;
  a.scores = nullptr;
  if (pl.ws_bytes > 0) {
    char *w = static_cast<char *>(ws);
    const size_t words = ((size_t)pl.n_problems * 4 + 255) & ~(size_t)255;
    a.counters = reinterpret_cast<uint32_t *>(w);
    a.failed = reinterpret_cast<uint32_t *>(w + words);
    a.stats = reinterpret_cast<float2 *>(w + 2 * words);
    a.scores = reinterpret_cast<float *>(w + 2 * words +
                                         (((size_t)pl.n_problems * pl.n_chunks * nf * 8 + 255) & ~(size_t)255));
  }
  // Kc (or window keys) [B*G][NR][d] as a 3-D map (d, NR, B*G), 64 x 128-row boxes
  CUtensorMap mK;
  const uint64_t kdim[3] = {(uint64_t)kD, (uint64_t)a.NR, (uint64_t)pl.n_problems};
  const uint64_t kstr[2] = {(uint64_t)kD * 2, (uint64_t)a.NR * kD * 2};
  const uint32_t kbox[3] = {64, kPieceRows, 1};
  if (a.NR < 1 || !tc::make_map_nd(&mK, kc, 3, kdim, kstr, kbox)) return cudaErrorNotSupported;
  const size_t smem = 1024 + (size_t)kRing * kPieceBytes + kHsmOpB +
                      (size_t)std::max(pl.ncand_max, 1) * 4;
  // the head count rounded up to a power of two fixes the unrolling
  const int nft_i = nf <= 1 ? 0 : nf <= 2 ? 1 : nf <= 4 ? 2 : nf <= 8 ? 3 : 4;
  void (*const kerns[2][5])(CUtensorMap, HsmArgs) = {
      {hsm_select_kernel<1, 1>, hsm_select_kernel<1, 2>, hsm_select_kernel<1, 4>,
       hsm_select_kernel<1, 8>, hsm_select_kernel<1, 16>},
      {hsm_select_kernel<4, 1>, hsm_select_kernel<4, 2>, hsm_select_kernel<4, 4>,
       hsm_select_kernel<4, 8>, hsm_select_kernel<4, 16>}};
  auto kern = kerns[pool == 1 ? 0 : 1][nft_i];
  {
    static size_t raised[2][5][64] = {{{0}}};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    size_t &r = raised[pool == 1 ? 0 : 1][nft_i][dev];
    if (r < smem) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e != cudaSuccess) return e;
      r = smem;
    }
  }
  const long long grid = pl.n_problems * pl.n_chunks;
  const cudaError_t e = launch_pdl(kern, (unsigned)grid, kSelThreads, smem, stream, mK, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sparda
