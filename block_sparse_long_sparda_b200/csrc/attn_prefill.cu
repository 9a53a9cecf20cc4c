// attn_prefill.cu -- block-sparse prefill attention: every token of a query
// chunk attends over the keys of its own block set, causal.
//
// Pages cited: [p4 <section>] = the article "SparDA: a fourth projection that
// lets sparse attention prefetch its own KV cache" (ai.thesatyajit.com);
// [p1 <section>] = the SparDA summary page at deepresearch2agi.pages.dev.
//
// [p4 "The fourth projection", Algorithm 1 / Eq. 5]: O_l = attention(Q_l,
// K_l[B_l], V_l[B_l]) with every key resident on the GPU, each query token
// with its own set B_l(i) (init U local U top-k, per token and group).
//
// Design (B200): block-major.  With per-token sets, the tokens that chose a
// block are scattered over the whole chunk (each block of a 128K sequence is
// picked by ~64 of 2048 tokens), so streaming each token's own list reads
// every block ~17 times through L2.  Here every selected block's K/V is read
// once per (sequence, group) for all the tokens that chose it:
//  1. invert_kernel -- one CTA per (sequence, group): the token -> blocks
//     lists become block -> tokens lists (a counting sort in shared
//     memory), and the blocks are cut into work items of up to 128 / R * 4
//     tokens (four 128-row tiles);
//  2. attn_block_kernel -- persistent, one CTA per SM.  A producer warp takes
//     items from a global counter and brings the block's K and V by TMA
//     (128-byte swizzle, no multicast) into a three-stage ring.  A tile is
//     128 rows = (token, head) pairs of the item; two warpgroups of row
//     threads take alternate tiles: each gathers its tile's query rows
//     (cp.async, straight into the swizzled operand), and after one
//     thread has issued S = Q K^T (tcgen05, M = 128, N = 64, K = 128, fp32
//     in TMEM) it runs the row softmax over the block's 64 keys (exp2
//     domain, causal inside the token's own block) and writes P (bf16); after
//     O = P V (M = 128, N = 128, K = 64) it writes the row's partial: o / l
//     in fp16 and (m, l) in fp32, at the (token, group, set position, head)
//     slot.  The two warpgroups ping-pong on the tensor core, and each
//     gathers its next tile's rows while its current product runs;
//  3. merge_kernel -- one warp per (token, group): for each head the
//     partials of the token's set combine as o = sum_s l_s 2^(m_s - M) o_s /
//     sum_s l_s 2^(m_s - M), M = max_s m_s.
// Every wait is bounded; a timeout sets SPARDA_DEV_TIMEOUT, drains what was
// issued and frees TMEM.  Shapes the block-major path does not take (more
// than 16384 blocks, more than 2^21 query tokens, sets of 2048 entries or
// more), or sparda_tuning::attn_prefill_per_token, use the per-token gather
// kernel of attn_decode.cu instead.
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace sparda {

namespace {

constexpr int kRows = 128;            // rows (token, head) per tile: the MMA's M
constexpr int kTilesPerItem = 4;      // tiles of one item share its K/V stage
constexpr int kSBits = 11;            // list entry = token << kSBits | set position
constexpr int kMaxSetEntries = (1 << kSBits) - 1;
constexpr int kMaxTokens = 1 << (32 - kSBits);
constexpr int kInvThreads = 1024;
constexpr int kMaxBlocksInv = 16384;  // blocks per sequence the inversion holds in shared memory
constexpr int kNst = 3;               // K/V ring stages (32 KB each)
constexpr int kTileRing = 8;          // tile descriptors in flight
constexpr int kBlkThreads = 320;      // 2 row warpgroups, producer, MMA issuer
constexpr int kWarpProd = 8, kWarpMma = 9;
constexpr int kTile8 = 8192;          // 64 rows x 64 bf16, one swizzled tile
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// 1. block -> tokens lists and work items
// ---------------------------------------------------------------------------
struct InvArgs {
  const int32_t *idx;      // [B][nq][G][S]
  const int32_t *seq_len;
  int32_t *status;
  uint32_t *list;          // [B*G][nq*S]: token << kSBits | s, grouped by block
  int4 *items;             // {bg, block, first list entry, tokens}
  uint32_t *counters;      // [0] items written, [1] items taken (block pass)
  int B, G, nq, S, NB, T, q_start, tpi;
};

// exclusive prefix sums of two per-thread values over the CTA; returns the
// totals in tot0/tot1
__device__ void block_scan2(uint32_t v0, uint32_t v1, uint32_t &x0, uint32_t &x1, uint32_t &tot0,
                            uint32_t &tot1, uint32_t *tmp /* [2][33] */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t a = v0, b = v1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t ta = __shfl_up_sync(0xffffffffu, a, o), tb = __shfl_up_sync(0xffffffffu, b, o);
    if (lane >= o) {
      a += ta;
      b += tb;
    }
  }
  if (lane == 31) {
    tmp[warp] = a;
    tmp[33 + warp] = b;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t wa = tmp[lane], wb = tmp[33 + lane];
    uint32_t ia = wa, ib = wb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t ta = __shfl_up_sync(0xffffffffu, ia, o), tb = __shfl_up_sync(0xffffffffu, ib, o);
      if (lane >= o) {
        ia += ta;
        ib += tb;
      }
    }
    tmp[lane] = ia - wa;
    tmp[33 + lane] = ib - wb;
    if (lane == 31) {
      tmp[32] = ia;
      tmp[65] = ib;
    }
  }
  __syncthreads();
  x0 = tmp[warp] + a - v0;
  x1 = tmp[33 + warp] + b - v1;
  tot0 = tmp[32];
  tot1 = tmp[65];
  __syncthreads();
}

__global__ void __launch_bounds__(kInvThreads) invert_kernel(InvArgs a) {
  extern __shared__ uint32_t cnt[];  // [NB]: counts, then write cursors
  __shared__ uint32_t tmp[66];
  __shared__ uint32_t s_base;
  const int tid = threadIdx.x;
  const int bg = blockIdx.x, b = bg / a.G, g = bg % a.G;
  pdl_trigger();
  pdl_wait();
  int qs = a.q_start;
  if (a.seq_len) {  // the chunk is the sequence's last nq tokens; an invalid length has no work
    const int len = a.seq_len[b];
    if (len < a.nq || len > a.T) return;
    qs = len - a.nq;
  }
  for (int j = tid; j < a.NB; j += kInvThreads) cnt[j] = 0u;
  __syncthreads();
  const uint32_t E = (uint32_t)a.nq * (uint32_t)a.S;  // < 2^32 (nq < 2^21, S < 2^11)
  const int32_t *idx_bg = a.idx + (long long)b * a.nq * a.G * a.S + (long long)g * a.S;
  const long long tok_stride = (long long)a.G * a.S;
  // entry e of (b, g): token e / S, set position e % S; four loads in flight per thread
  auto load4 = [&](uint32_t e0, int (&j)[4], int (&i)[4], int (&sp)[4]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t e = e0 + (uint32_t)q * kInvThreads;
      i[q] = (int)(e / (uint32_t)a.S);
      sp[q] = (int)(e - (uint32_t)i[q] * (uint32_t)a.S);
      j[q] = e < E ? __ldg(idx_bg + i[q] * tok_stride + sp[q]) : -1;
    }
  };
  bool bad = false;
  for (uint32_t e0 = tid; e0 < E; e0 += 4u * kInvThreads) {
    int j[4], i[4], sp[4];
    load4(e0, j, i, sp);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (j[q] < 0) continue;
      if (j[q] >= a.NB || j[q] > (qs + i[q]) / kBlk) {  // not a block this token may attend to
        bad = true;
        continue;
      }
      atomicAdd(&cnt[j[q]], 1u);
    }
  }
  if (__syncthreads_or(bad) && tid == 0) flag_status(a.status, SPARDA_DEV_RANGE);
  // list start and item offset of every block (each thread a run of blocks)
  const int per = (a.NB + kInvThreads - 1) / kInvThreads;
  const int j0 = min(a.NB, tid * per), j1 = min(a.NB, j0 + per);
  uint32_t sum_t = 0, sum_i = 0;
  for (int j = j0; j < j1; ++j) {
    sum_t += cnt[j];
    sum_i += (cnt[j] + a.tpi - 1) / a.tpi;
  }
  uint32_t off_t, off_i, tot_t, tot_i;
  block_scan2(sum_t, sum_i, off_t, off_i, tot_t, tot_i, tmp);
  if (tid == 0) s_base = atomicAdd(&a.counters[0], tot_i);
  __syncthreads();
  const uint32_t base = s_base;
  for (int j = j0; j < j1; ++j) {
    const uint32_t c = cnt[j];
    for (uint32_t k = 0; k * a.tpi < c; ++k)
      a.items[base + off_i + k] = make_int4(bg, j, (int)(off_t + k * a.tpi),
                                            (int)min((uint32_t)a.tpi, c - k * a.tpi));
    off_i += (c + a.tpi - 1) / a.tpi;
    cnt[j] = off_t;  // the block's write cursor
    off_t += c;
  }
  __syncthreads();
  uint32_t *list = a.list + (long long)bg * E;
  for (uint32_t e0 = tid; e0 < E; e0 += 4u * kInvThreads) {
    int j[4], i[4], sp[4];
    load4(e0, j, i, sp);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (j[q] < 0 || j[q] >= a.NB || j[q] > (qs + i[q]) / kBlk) continue;
      const uint32_t p = atomicAdd(&cnt[j[q]], 1u);
      list[p] = ((uint32_t)i[q] << kSBits) | (uint32_t)sp[q];
    }
  }
}

// ---------------------------------------------------------------------------
// 2. the block pass
// ---------------------------------------------------------------------------
struct BlkArgs {
  const uint16_t *Q;        // [B][nq][Hq][d]
  const uint32_t *list;
  const int4 *items;
  uint32_t *counters;
  float2 *ml;               // [B][nq][G][S][R] (m, l) in the exp2 domain
  __half *po;               // [B][nq][G][S][R][d] o / l
  const int32_t *seq_len;
  int32_t *status;
  long long bg_rows;        // K/V rows per (sequence, group)
  int B, G, nq, S, NB, T, q_start, R, rshift;
  float scale_log2;
  long long wait_cycles;
};

struct TileDesc {
  int bg, j, n_rows;        // (sequence, group), block, valid rows of the tile
  int stage, kv_par, last;  // K/V stage, its phase bit, last tile of the item
  int end;                  // no more tiles
  uint32_t ent[kRows];      // list entries of the tile's tokens (token << kSBits | s)
};

// where a row's query comes from and where its partial goes (null: no row)
struct RowAddr {
  const uint16_t *src;
  __half *dst;
};

struct BlkCtl {
  uint64_t kv_full[kNst], kv_empty[kNst];
  uint64_t t_full[kTileRing], t_empty[kTileRing];
  uint64_t a_ready[2], s_full[2], p_full[2], o_full[2];
  TileDesc desc[kTileRing];
  RowAddr rows[2][2][kRows];  // [warpgroup][tile parity][row]
  uint32_t tmem_base;
  int s_abort;
};

// K/V ring | two query-row tiles (32 KB) | two P tiles (16 KB) | control
constexpr size_t kBlkSmem = (size_t)kNst * 4 * kTile8 + 2 * 32768 + 2 * 16384 +
                            (sizeof(BlkCtl) + 127) / 128 * 128;

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      *abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__global__ void __launch_bounds__(kBlkThreads, 1)
    attn_block_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                      BlkArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *kv = smem_raw;                          // kNst x [K lo | V lo | K hi | V hi]
  uint8_t *qa = kv + kNst * 4 * kTile8;            // 2 x [2 dim halves][128 rows][64]
  uint8_t *pa = qa + 2 * 32768;                    // 2 x [128 rows][64 keys]
  BlkCtl &ctl = *reinterpret_cast<BlkCtl *>(pa + 2 * 16384);
  volatile int *s_abort = &ctl.s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long lim = a.wait_cycles;
  pdl_trigger();
  if (smem_addr(smem_raw) & 1023u) {  // the swizzled tiles would be misread
    pdl_wait();
    if (tid == 0) flag_status(a.status, SPARDA_DEV_LAYOUT);
    return;
  }
  if (tid == 0) {
    for (int s = 0; s < kNst; ++s) {
      mbar_init(&ctl.kv_full[s], 1);
      mbar_init(&ctl.kv_empty[s], 1);
    }
    for (int q = 0; q < kTileRing; ++q) {
      mbar_init(&ctl.t_full[q], 1);
      mbar_init(&ctl.t_empty[q], kRows + 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&ctl.a_ready[w], kRows);
      mbar_init(&ctl.s_full[w], 1);
      mbar_init(&ctl.p_full[w], kRows);
      mbar_init(&ctl.o_full[w], 1);
    }
    *s_abort = 0;
    fence_mbar_init();
    tc::prefetch_map(&mapK);
    tc::prefetch_map(&mapV);
  }
  // TMEM: per warpgroup two 128-column regions, alternating by tile; a
  // tile's S takes the first 64 columns of its region and its O (written
  // after the softmax has read S) all 128
  if (warp == 0) tc::tmem_alloc(&ctl.tmem_base, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ctl.tmem_base;
  pdl_wait();  // the lists and items of the inversion are complete

  int produced = 0;                // producer: items whose K/V loads were issued
  int issued_s = 0, issued_p = 0;  // MMA issuer: products committed

  if (warp == kWarpProd) {
    // ====== producer (whole warp): items -> K/V stages and tile descriptors ======
    // Lane 0 takes items (two per atomic, the next pair requested while the
    // current one is set up) and issues the TMA; the warp copies each item's
    // list entries straight into its tiles' descriptors, so the row threads
    // find them in shared memory.
    const uint32_t n_items = __ldcg(&a.counters[0]);
    const int tshift = 7 - a.rshift;  // tokens per tile = 128 / R = 1 << tshift
    const long long E = (long long)a.nq * a.S;
    int u = 0;
    bool ok = true;
    uint32_t it0 = 0;
    if (lane == 0) it0 = atomicAdd(&a.counters[1], 2u);
    it0 = __shfl_sync(0xffffffffu, it0, 0);
#pragma unroll 1
    while (ok && it0 < n_items) {
      uint32_t it_next = 0;
      if (lane == 0) it_next = atomicAdd(&a.counters[1], 2u);  // used one round later
      int4 recs[2];  // both records load together
#pragma unroll
      for (int q = 0; q < 2; ++q)
        recs[q] = it0 + q < n_items ? __ldcg(&a.items[it0 + q]) : make_int4(0, 0, 0, 0);
#pragma unroll 1
      for (uint32_t it = it0; it < min(it0 + 2u, n_items) && ok; ++it) {
        const int4 rec = it == it0 ? recs[0] : recs[1];
        const int st = produced % kNst;
        bool f = true;
        if (lane == 0 && produced >= kNst)
          f = wait_bar(&ctl.kv_empty[st], (uint32_t)(((produced / kNst) - 1) & 1), s_abort, lim);
        if (!__shfl_sync(0xffffffffu, (int)f, 0)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t *dst = kv + st * 4 * kTile8;
          const int row = (int)((long long)rec.x * a.bg_rows + (long long)rec.y * kBlk);
          mbar_arrive_expect_tx(&ctl.kv_full[st], 4 * kTile8);
          tc::tma_load_2d(dst, &mapK, 0, row, &ctl.kv_full[st]);
          tc::tma_load_2d(dst + kTile8, &mapV, 0, row, &ctl.kv_full[st]);
          tc::tma_load_2d(dst + 2 * kTile8, &mapK, 64, row, &ctl.kv_full[st]);
          tc::tma_load_2d(dst + 3 * kTile8, &mapV, 64, row, &ctl.kv_full[st]);
        }
        const int kv_par = (produced / kNst) & 1;
        ++produced;
        const int n_tiles = (rec.w + (1 << tshift) - 1) >> tshift;
        // the item's tiles need free descriptor slots
        for (int m = 0; m < n_tiles; ++m) {
          const int v = u + m;
          bool fr = true;
          if (lane == 0 && v >= kTileRing)
            fr = wait_bar(&ctl.t_empty[v % kTileRing], (uint32_t)(((v / kTileRing) - 1) & 1), s_abort, lim);
          if (!__shfl_sync(0xffffffffu, (int)fr, 0)) {
            ok = false;
            break;
          }
        }
        if (!ok) break;
        const uint32_t *src = a.list + (long long)rec.x * E + rec.z;
#pragma unroll 4
        for (int e = lane; e < rec.w; e += 32)
          ctl.desc[(u + (e >> tshift)) % kTileRing].ent[e & ((1 << tshift) - 1)] = __ldg(src + e);
        if (lane == 0) {
          for (int m = 0; m < n_tiles; ++m) {
            TileDesc &d = ctl.desc[(u + m) % kTileRing];
            d.bg = rec.x;
            d.j = rec.y;
            d.n_rows = min(1 << tshift, rec.w - (m << tshift)) << a.rshift;
            d.stage = st;
            d.kv_par = kv_par;
            d.last = m == n_tiles - 1;
            d.end = 0;
          }
        }
        __syncwarp();  // the lanes' entries are written before lane 0 publishes the tiles
        if (lane == 0)
          for (int m = 0; m < n_tiles; ++m) mbar_arrive(&ctl.t_full[(u + m) % kTileRing]);
        u += n_tiles;
      }
      it0 = __shfl_sync(0xffffffffu, it_next, 0);
    }
    // one end marker for each row warpgroup
    for (int e = 0; e < 2 && ok; ++e) {
      bool fr = true;
      if (lane == 0 && u >= kTileRing)
        fr = wait_bar(&ctl.t_empty[u % kTileRing], (uint32_t)(((u / kTileRing) - 1) & 1), s_abort, lim);
      if (!__shfl_sync(0xffffffffu, (int)fr, 0)) {
        ok = false;
        break;
      }
      if (lane == 0) {
        ctl.desc[u % kTileRing].end = 1;
        mbar_arrive(&ctl.t_full[u % kTileRing]);
      }
      ++u;
    }
    if (!ok && lane == 0) *s_abort = 1;
  } else if (warp == kWarpMma) {
    // ====== MMA issuer: S(u) and P V(v), each in tile order, whichever is ready ======
    // S(u) needs the tile's descriptor, its K/V stage and its query rows; the
    // row warpgroup hands those in only after it has read S and O of its
    // previous tile, so S and O of a warpgroup are never overwritten early.
    if (lane == 0) {
      constexpr uint32_t id_s = tc::idesc_bf16(128, 64, false, false);
      constexpr uint32_t id_o = tc::idesc_bf16(128, 128, false, true);
      int n_s = 0, n_p = 0, total = -1;  // S issued, PV issued, tiles (once the end is seen)
      long long t0 = clock64();
      bool ok = true;
#pragma unroll 1
      while (total < 0 || n_p < total) {
        bool moved = false;
        if (total < 0 && n_s - n_p < 4) {
          const int q = n_s % kTileRing, w = n_s & 1;
          const uint32_t reg = (uint32_t)(w * 256 + ((n_s >> 1) & 1) * 128);  // the tile's TMEM region
          if (mbar_test_wait(&ctl.t_full[q], (uint32_t)((n_s / kTileRing) & 1))) {
            if (ctl.desc[q].end) {
              total = n_s;
              moved = true;
            } else if (mbar_test_wait(&ctl.kv_full[ctl.desc[q].stage], (uint32_t)ctl.desc[q].kv_par) &&
                       mbar_test_wait(&ctl.a_ready[w], (uint32_t)((n_s >> 1) & 1))) {
              const int st = ctl.desc[q].stage;
              tc::fence_after_sync();
              const uint64_t dA = tc::sdesc(qa + w * 32768, 16, 1024);
              const uint64_t dK = tc::sdesc(kv + st * 4 * kTile8, 16, 1024);
#pragma unroll
              for (int k = 0; k < 8; ++k)
                tc::mma_bf16(tmem + reg, dA + (uint64_t)((k >> 2) * (16384 >> 4) + (k & 3) * 2),
                             dK + (uint64_t)((k >> 2) * (2 * kTile8 >> 4) + (k & 3) * 2), id_s, k > 0);
              tc::mma_commit(&ctl.s_full[w]);
              issued_s = ++n_s;
              moved = true;
            }
          }
        }
        if (n_p < n_s) {
          const int q = n_p % kTileRing, w = n_p & 1;
          const uint32_t reg = (uint32_t)(w * 256 + ((n_p >> 1) & 1) * 128);
          if (mbar_test_wait(&ctl.p_full[w], (uint32_t)((n_p >> 1) & 1))) {
            tc::fence_after_sync();
            // the tile's descriptor stays in its slot until this product is issued
            const int st = ctl.desc[q].stage;
            const uint64_t dP = tc::sdesc(pa + w * 16384, 16, 1024);
            const uint64_t dV = tc::sdesc(kv + st * 4 * kTile8 + kTile8, 2 * kTile8, 1024);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc::mma_bf16(tmem + reg, dP + (uint64_t)(k * 2), dV + (uint64_t)(k * 128), id_o, k > 0);
            tc::mma_commit(&ctl.o_full[w]);
            if (ctl.desc[q].last) tc::mma_commit(&ctl.kv_empty[st]);
            mbar_arrive(&ctl.t_empty[q]);
            issued_p = ++n_p;
            moved = true;
          }
        }
        if (moved) {
          t0 = clock64();
          continue;
        }
        if (*s_abort) {
          ok = false;
          break;
        }
        if (clock64() - t0 > lim) {
          ok = false;
          break;
        }
        __nanosleep(32);
      }
      if (!ok) *s_abort = 1;
    }
  } else {
    // ====== row warpgroups (warps 0-3: tiles 0, 2, ...; 4-7: 1, 3, ...) ======
    // Thread r owns row r (TMEM lane r) for the softmax; the loads of query
    // rows and the stores of partials are done by whole warps over their 32
    // rows, eight lanes per 128-byte half row, so every access is whole lines.
    const int w = warp >> 2, wq = warp & 3;
    const int r = tid & 127;                     // row of the tile = TMEM lane
    const uint32_t lane_sel = (uint32_t)(wq * 32) << 16;
    uint8_t *A = qa + w * 32768;
    uint8_t *P = pa + w * 16384;
    const int R = a.R;
    const int h = r & (R - 1);
    bool ok = true;
    struct Row {
      int end, valid, j, pos;
      long long slot;
    };
    // the tile's descriptor -> this row's token; its addresses go to the
    // warpgroup's row table (parity par) for the warp-wide loads and stores
    auto read_desc = [&](int u, int par, Row &row) -> bool {
      const int q = u % kTileRing;
      if (!wait_bar(&ctl.t_full[q], (uint32_t)((u / kTileRing) & 1), s_abort, lim)) return false;
      const TileDesc &d = ctl.desc[q];
      row.end = d.end;
      if (d.end) return true;
      row.valid = r < d.n_rows;
      row.j = d.j;
      const int bg = d.bg, b = bg / a.G, g = bg - b * a.G;
      const uint32_t e = row.valid ? d.ent[r >> a.rshift] : 0u;
      mbar_arrive(&ctl.t_empty[q]);
      const int i = (int)(e >> kSBits), s = (int)(e & kMaxSetEntries);
      int qs = a.q_start;
      if (a.seq_len) qs = __ldg(&a.seq_len[b]) - a.nq;  // valid lengths only reach here
      row.pos = qs + i;
      const long long tok = (long long)b * a.nq + i;
      row.slot = ((tok * a.G + g) * a.S + s) * (long long)R + h;
      RowAddr ra;
      ra.src = row.valid ? a.Q + (tok * a.G + g) * (long long)R * kD + (long long)h * kD : nullptr;
      ra.dst = row.valid ? a.po + row.slot * kD : nullptr;
      ctl.rows[w][par][r] = ra;
      return true;
    };
    // the warp's 32 query rows of the tile (parity par) into the swizzled A tile
    auto gather = [&](int par) {
      __syncwarp();  // the warp's row table entries are written
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int rr = wq * 32 + t * 4 + (lane >> 3), c = lane & 7;
        const uint16_t *src = ctl.rows[w][par][rr].src;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
          cp_async16(A + hf * 16384 + tc::sw128_offset(rr, c * 8), src ? src + hf * 64 + c * 8 : a.Q,
                     src ? 16u : 0u);
      }
      cp_async_commit();
    };
    int u = w, k = 0;
    Row cur{}, nxt{};
    ok = __all_sync(0xffffffffu, read_desc(u, 0, cur));
    if (ok && !cur.end) {
      gather(0);
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(&ctl.a_ready[w]);
    }
#pragma unroll 1
    while (ok && !cur.end) {
      // ---- S(u) is done: A is free, so the next tile's query rows start loading ----
      ok = wait_bar(&ctl.s_full[w], (uint32_t)(k & 1), s_abort, lim);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ok = __all_sync(0xffffffffu, read_desc(u + 2, (k + 1) & 1, nxt));
      if (!ok) break;
      if (!nxt.end) gather((k + 1) & 1);
      // ---- softmax of the row over the block's keys -> P ----
      tc::fence_after_sync();
      const uint32_t reg = tmem + (uint32_t)(w * 256 + (k & 1) * 128) + lane_sel;  // S(u), then O(u)
      const int lim_key = cur.pos - cur.j * kBlk;  // keys after the token are masked
      float sv[64];
      tc::tmem_ld64(reg, sv);
      float m;
      {
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (lim_key >= kBlk - 1) {  // a block before the token's own: every key counts
#pragma unroll
          for (int c = 0; c < 64; ++c) mq[c & 3] = fmaxf(mq[c & 3], sv[c]);
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c <= lim_key) mq[c & 3] = fmaxf(mq[c & 3], sv[c]);
        }
        m = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * a.scale_log2;
      }
      // a row with no token (past the tile's rows) gets P = 0: exp2(x - inf)
      const float msub = cur.valid ? m : INFINITY;
      float lq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kk = c8 * 8 + 2 * e;
          const float x0 = kk <= lim_key ? fmaf(sv[kk], a.scale_log2, -msub) : -INFINITY;
          const float x1 = kk + 1 <= lim_key ? fmaf(sv[kk + 1], a.scale_log2, -msub) : -INFINITY;
          const __nv_bfloat162 pb = __floats2bfloat162_rn(tc::ex2_approx(x0), tc::ex2_approx(x1));
          lq[e] += __low2float(pb) + __high2float(pb);
          pk[e] = *reinterpret_cast<const uint32_t *>(&pb);
        }
        *reinterpret_cast<uint4 *>(P + tc::sw128_offset(r, c8 * 8)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      const float l = (lq[0] + lq[1]) + (lq[2] + lq[3]);
      fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(&ctl.p_full[w]);
      // ---- the next tile's query rows go to the MMA issuer now, so its S
      // runs (in the other TMEM region) while P V(u) and the epilogue do ----
      if (!nxt.end) {
        cp_async_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(&ctl.a_ready[w]);
      }
      // ---- P V(u) -> the partials, staged through P (free once P V is done) ----
      ok = wait_bar(&ctl.o_full[w], (uint32_t)(k & 1), s_abort, lim);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc::fence_after_sync();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      uint8_t *stg = P + wq * 4096;  // the warp's 32 rows x 128 bytes
      const int par = k & 1;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float o[64];
        tc::tmem_ld64(reg + hf * 64, o);
        // this lane's half row -> staging (chunks rotated by row: no bank conflicts)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t hv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __half2 hh = __floats2half2_rn(o[c * 8 + 2 * e] * inv_l, o[c * 8 + 2 * e + 1] * inv_l);
            hv[e] = *reinterpret_cast<const uint32_t *>(&hh);
          }
          *reinterpret_cast<uint4 *>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
              make_uint4(hv[0], hv[1], hv[2], hv[3]);
        }
        __syncwarp();
        // whole 128-byte lines out: eight lanes per row, four rows per store
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int rl = t * 4 + (lane >> 3), c = lane & 7;
          const uint4 v = *reinterpret_cast<const uint4 *>(stg + rl * 128 + ((c ^ (rl & 7)) << 4));
          __half *dst = ctl.rows[w][par][wq * 32 + rl].dst;
          if (dst) *reinterpret_cast<uint4 *>(dst + hf * 64 + c * 8) = v;
        }
        __syncwarp();  // staging is reused by the next half
      }
      if (cur.valid) a.ml[cur.slot] = make_float2(m, l);
      tc::fence_before_sync();
      cur = nxt;
      u += 2;
      ++k;
    }
    cp_async_wait_all();  // no copy may still target the tiles when the CTA leaves
    if (!ok) *s_abort = 1;
  }

  __syncthreads();
  if (*s_abort) {
    flag_status(a.status, SPARDA_DEV_TIMEOUT);
    // let what was issued land or finish (bounded) before the memory is released
    if (warp == kWarpProd && lane == 0)
      for (int v = max(0, produced - kNst); v < produced; ++v)
        (void)mbar_wait_bounded(&ctl.kv_full[v % kNst], (uint32_t)((v / kNst) & 1));
    if (warp == kWarpMma && lane == 0) {
      for (int v = max(0, issued_s - 2); v < issued_s; ++v)
        (void)mbar_wait_bounded(&ctl.s_full[v & 1], (uint32_t)((v >> 1) & 1));
      for (int v = max(0, issued_p - 2); v < issued_p; ++v)
        (void)mbar_wait_bounded(&ctl.o_full[v & 1], (uint32_t)((v >> 1) & 1));
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// 3. merge of each token's partials
// ---------------------------------------------------------------------------
struct MergeArgs {
  const int32_t *idx;       // [B][nq][G][S]
  const float2 *ml;
  const __half *po;
  uint16_t *O;              // [B][nq][Hq][d]
  const int32_t *seq_len;
  int32_t *status;
  int B, G, nq, S, NB, T, q_start, R;
};

constexpr int kMergeWarps = 8;

// One warp per (token, group, head); lane = 4 output dims.  The loads of
// eight set entries are in flight together; a slot no valid entry wrote is
// loaded too (it lies inside the workspace) but selected away, never used.
__global__ void __launch_bounds__(kMergeWarps * 32) merge_kernel(MergeArgs a) {
  const int lane = threadIdx.x & 31;
  const long long wi = (long long)blockIdx.x * kMergeWarps + (threadIdx.x >> 5);  // (b, i, g, h)
  pdl_trigger();
  pdl_wait();
  const int R = a.R;
  if (wi >= (long long)a.B * a.nq * a.G * R) return;
  const int h = (int)(wi % R);
  const long long pr = wi / R;  // (b, i, g)
  const int g = (int)(pr % a.G);
  const long long tok = pr / a.G;
  const int i = (int)(tok % a.nq), b = (int)(tok / a.nq);
  uint16_t *out = a.O + (pr * R + h) * (long long)kD;
  int qs = a.q_start;
  if (a.seq_len) {
    const int len = a.seq_len[b];
    if (len < a.nq || len > a.T) {  // an invalid length: a zero output
      reinterpret_cast<uint2 *>(out)[lane] = make_uint2(0, 0);
      if (lane == 0 && i == 0 && g == 0 && h == 0) flag_status(a.status, SPARDA_DEV_RANGE);
      return;
    }
    qs = len - a.nq;
  }
  const int c = (qs + i) / kBlk;
  const int32_t *ids = a.idx + pr * a.S;
  const float2 *ml = a.ml + pr * (long long)a.S * R + h;
  const __half *po = a.po + (pr * a.S * R + h) * (long long)kD + lane * 4;
  const long long po_stride = (long long)R * kD;
  float M = -INFINITY;
  for (int s = lane; s < a.S; s += 32) {
    const int j = __ldg(ids + s);
    if (j >= 0 && j < a.NB && j <= c) M = fmaxf(M, ml[(long long)s * R].x);
  }
  M = warp_max_xor(M, 1, 32);
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f, L = 0.f;
#pragma unroll 1
  for (int s0 = 0; s0 < a.S; s0 += 32) {
    const int s = s0 + lane;
    float wgt = 0.f;
    if (s < a.S) {
      const int j = __ldg(ids + s);
      if (j >= 0 && j < a.NB && j <= c) {
        const float2 v = ml[(long long)s * R];
        wgt = v.y * exp2f(v.x - M);
      }
    }
    L += wgt;
    const int n = min(32, a.S - s0);
    const __half *p0 = po + (long long)s0 * po_stride;
    int q = 0;
#pragma unroll 1
    for (; q + 8 <= n; q += 8) {
      uint2 raw[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) raw[t] = __ldcs(reinterpret_cast<const uint2 *>(p0 + (long long)(q + t) * po_stride));
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float wq = __shfl_sync(0xffffffffu, wgt, q + t);
        const __half2 h0 = *reinterpret_cast<const __half2 *>(&raw[t].x);
        const __half2 h1 = *reinterpret_cast<const __half2 *>(&raw[t].y);
        if (wq != 0.f) {
          acc0 = fmaf(wq, __low2float(h0), acc0);
          acc1 = fmaf(wq, __high2float(h0), acc1);
          acc2 = fmaf(wq, __low2float(h1), acc2);
          acc3 = fmaf(wq, __high2float(h1), acc3);
        }
      }
    }
    for (; q < n; ++q) {
      const uint2 raw = __ldcs(reinterpret_cast<const uint2 *>(p0 + (long long)q * po_stride));
      const float wq = __shfl_sync(0xffffffffu, wgt, q);
      const __half2 h0 = *reinterpret_cast<const __half2 *>(&raw.x);
      const __half2 h1 = *reinterpret_cast<const __half2 *>(&raw.y);
      if (wq != 0.f) {
        acc0 = fmaf(wq, __low2float(h0), acc0);
        acc1 = fmaf(wq, __high2float(h0), acc1);
        acc2 = fmaf(wq, __low2float(h1), acc2);
        acc3 = fmaf(wq, __high2float(h1), acc3);
      }
    }
  }
  L = warp_sum_xor(L, 1, 32);
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const __nv_bfloat162 o0 = __floats2bfloat162_rn(acc0 * inv, acc1 * inv);
  const __nv_bfloat162 o1 = __floats2bfloat162_rn(acc2 * inv, acc3 * inv);
  uint2 st;
  st.x = *reinterpret_cast<const uint32_t *>(&o0);
  st.y = *reinterpret_cast<const uint32_t *>(&o1);
  reinterpret_cast<uint2 *>(out)[lane] = st;
}

// ---------------------------------------------------------------------------
// host: layout of the workspace, eligibility
// ---------------------------------------------------------------------------
struct BlkPlan {
  bool ok;
  int R, S, NB, tpi;
  long long max_items;
  size_t off_list, off_items, off_ml, off_po, total;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

BlkPlan plan_block(const sparda_params &p, int nq) {
  BlkPlan pl{};
  pl.R = p.Hq / p.G;
  pl.S = p.k + p.n_init + p.n_local;
  pl.NB = (p.T + kBlk - 1) / kBlk;
  pl.tpi = (kRows * kTilesPerItem) / pl.R;
  pl.ok = tuning(p).attn_prefill_per_token == 0 && pl.NB <= kMaxBlocksInv && nq < kMaxTokens &&
          pl.S <= kMaxSetEntries;
  if (!pl.ok) return pl;
  const long long bgs = (long long)p.B * p.G;
  const long long entries = bgs * nq * pl.S;  // list entries and partial slots per head
  pl.max_items = bgs * (ceil_div_ll((long long)nq * pl.S, pl.tpi) + pl.NB);
  size_t off = 256;                                           // two counters
  pl.off_list = off;
  off += align256((size_t)entries * 4);
  pl.off_items = off;
  off += align256((size_t)pl.max_items * 16);
  pl.off_ml = off;
  off += align256((size_t)entries * pl.R * 8);
  pl.off_po = off;
  off += align256((size_t)entries * pl.R * kD * 2);
  pl.total = off;
  return pl;
}

}  // namespace

size_t prefill_ws_bytes(const sparda_params &p, int nq) {
  const BlkPlan pl = plan_block(p, nq);
  if (pl.ok) return pl.total;
  return plan_gather(p, (long long)p.B * nq * p.G).ws_bytes;
}

cudaError_t launch_attn_prefill(const sparda_params &p, const uint16_t *Q, int nq, int q_start,
                                const uint16_t *K, const uint16_t *V, long long bg_stride,
                                long long tok_stride, const int32_t *idx, uint16_t *O, void *ws,
                                size_t ws_bytes, int32_t *dev_status, cudaStream_t stream) {
  (void)ws_bytes;
  const BlkPlan pl = plan_block(p, nq);
  if (!pl.ok) {  // the per-token gather kernel
    const DecodePlan gp = plan_gather(p, (long long)p.B * nq * p.G);
    return launch_gather_attn(p, gp, nq, q_start, Q, K, V, bg_stride, (long long)kBlk * tok_stride,
                              idx, SPARDA_ADDR_LOGICAL, O, ws, dev_status, stream);
  }
  if ((long long)p.B * nq * p.G == 0) return cudaSuccess;
  char *w = static_cast<char *>(ws);
  uint32_t *counters = reinterpret_cast<uint32_t *>(w);
  cudaError_t e = cudaMemsetAsync(counters, 0, 8, stream);
  if (e != cudaSuccess) return e;
  // ---- 1. inversion ----
  InvArgs ia;
  ia.idx = idx;
  ia.seq_len = p.seq_len;
  ia.status = dev_status;
  ia.list = reinterpret_cast<uint32_t *>(w + pl.off_list);
  ia.items = reinterpret_cast<int4 *>(w + pl.off_items);
  ia.counters = counters;
  ia.B = p.B;
  ia.G = p.G;
  ia.nq = nq;
  ia.S = pl.S;
  ia.NB = pl.NB;
  ia.T = p.T;
  ia.q_start = q_start;
  ia.tpi = pl.tpi;
  const size_t inv_smem = (size_t)pl.NB * 4;
  struct Cached {
    void *ctx;
    int n_sm;
  };
  static Cached cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  void *ctx = current_context();
  if (cache[dev].n_sm == 0 || cache[dev].ctx != ctx) {
    int n_sm = 148;
    (void)cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    e = cudaFuncSetAttribute(invert_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kMaxBlocksInv * 4);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kBlkSmem);
    if (e != cudaSuccess) return e;
    cache[dev].n_sm = n_sm;
    cache[dev].ctx = ctx;
  }
  e = launch_pdl(invert_kernel, (unsigned)(p.B * p.G), kInvThreads, inv_smem, stream, ia);
  if (e != cudaSuccess) return e;
  // ---- 2. the block pass ----
  const long long kv_pairs = (long long)p.B * p.G;
  const long long bg_rows = bg_stride / kD;
  long long extent = (kv_pairs - 1) * bg_rows + (long long)pl.NB * kBlk;
  extent = std::min(extent, kv_pairs * bg_rows);
  if (extent >= (1LL << 31)) return cudaErrorInvalidValue;
  CUtensorMap mk, mv;
  if (!tc::make_map_2d(&mk, K, kD, (uint64_t)extent, kD, 64, 64) ||
      !tc::make_map_2d(&mv, V, kD, (uint64_t)extent, kD, 64, 64))
    return cudaErrorNotSupported;
  BlkArgs ba;
  ba.Q = Q;
  ba.list = ia.list;
  ba.items = ia.items;
  ba.counters = counters;
  ba.ml = reinterpret_cast<float2 *>(w + pl.off_ml);
  ba.po = reinterpret_cast<__half *>(w + pl.off_po);
  ba.seq_len = p.seq_len;
  ba.status = dev_status;
  ba.bg_rows = bg_rows;
  ba.B = p.B;
  ba.G = p.G;
  ba.nq = nq;
  ba.S = pl.S;
  ba.NB = pl.NB;
  ba.T = p.T;
  ba.q_start = q_start;
  ba.R = pl.R;
  ba.rshift = __builtin_ctz((unsigned)pl.R);
  const float scale = p.scale > 0.f ? p.scale : 1.0f / sqrtf((float)p.d);
  ba.scale_log2 = scale * kLog2e;
  const sparda_tuning &tu = tuning(p);
  ba.wait_cycles = tu.attn_wait_cycles > 0 ? tu.attn_wait_cycles : kWaitCycles;
  e = launch_pdl(attn_block_kernel, (unsigned)cache[dev].n_sm, kBlkThreads, kBlkSmem, stream, mk,
                 mv, ba);
  if (e != cudaSuccess) return e;
  // ---- 3. merge ----
  MergeArgs ma;
  ma.idx = idx;
  ma.ml = ba.ml;
  ma.po = ba.po;
  ma.O = O;
  ma.seq_len = p.seq_len;
  ma.status = dev_status;
  ma.B = p.B;
  ma.G = p.G;
  ma.nq = nq;
  ma.S = pl.S;
  ma.NB = pl.NB;
  ma.T = p.T;
  ma.q_start = q_start;
  ma.R = pl.R;
  const long long rows = (long long)p.B * nq * p.G * pl.R;  // (token, group, head)
  e = launch_pdl(merge_kernel, (unsigned)ceil_div_ll(rows, kMergeWarps), kMergeWarps * 32, 0,
                 stream, ma);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sparda
