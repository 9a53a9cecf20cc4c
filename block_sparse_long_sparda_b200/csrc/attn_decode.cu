// attn_decode.cu -- GQA block-sparse attention of single query tokens over
// their own block lists (decode; also the per-token prefill path).
//
// Pages cited: [p4 <section>] = the article "SparDA: a fourth projection that
// lets sparse attention prefetch its own KV cache" (ai.thesatyajit.com);
// [p1 <section>] = the SparDA summary page at deepresearch2agi.pages.dev.
//
// [p4 "The fourth projection", Eq. 5 / Algorithm 2]: O_l = attention(Q_l,
// K_l[B_l], V_l[B_l]): each query head attends over the keys of its GQA
// group's selected blocks only; fp32 softmax, fp32 accumulation.
//
// Design (B200).  A selected block is 32 KB of K+V; the R query heads of a
// group share it, so each block is a pair of tiny dense contractions:
// S^T[64 keys x R] = K[64x128] Q^T and O^T[128 dims x R] += V^T P^T.  They run
// on the 5th-generation tensor cores (tcgen05, bf16 operands in shared
// memory, fp32 accumulators in TMEM), which leaves the CUDA cores only the
// softmax -- a few dozen instructions per thread per block -- so the kernel
// streams K/V at HBM speed instead of being bound by instruction issue:
//  - stream-K: the (query, group) "pairs" and their list entries are
//    flattened and cut into equal contiguous ranges, one per CTA, with a grid
//    of as many CTAs as stay resident (three per SM with a two-stage ring,
//    two with three stages) -- one wave.  A range may start or end inside a
//    pair; each piece of a pair is a "segment";
//  - launched as a programmatic dependent of the previous kernel: barriers
//    and tensor maps are set up before waiting for it; the entry list of a
//    range is then read by all threads at once and compacted with a block
//    scan (one global-load latency per CTA);
//  - TMA (cp.async.bulk.tensor, 128-byte swizzle, no multicast) stages each
//    block as [K lo-dims | V lo-dims | K hi-dims | V hi-dims] (8 KB each) in
//    an NSTAGE ring, the K and the V tiles of a slot with barriers of their
//    own (for blocks that come from L2, K is refilled once S^T has read it
//    and V once O^T has, so V waits less in the slot); the pair's query rows
//    are loaded into the S^T issuer's registers one segment ahead.  The
//    M = 128 MMA for S^T reads rows 0-63 = the block's keys; its rows 64-127
//    alias the V tiles (which may still be loading) and are never read back;
//  - one thread issues the MMAs (N = 16: the group's heads, zero padded);
//    softmax per head in the exp2 domain over the thread-per-key rows of
//    S^T; P^T goes to shared memory as a bf16 K-major operand (the sum of
//    probabilities uses the same rounded values); O^T is read back with one
//    thread per output dim and rescaled in registers;
//  - at the end of a segment a pair that a single CTA covers is normalised
//    and written at once, otherwise the segment's (max, sum, unnormalised
//    output) goes to the workspace and the last CTA to finish the pair
//    (atomic ticket, no waiting) combines them.
// Every wait (TMA, MMA completion) is bounded: a timeout sets
// SPARDA_DEV_TIMEOUT, the CTA drains what it issued (bounded), frees its
// TMEM and leaves.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace sparda {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kGridMax = 3 * 148;               // most CTAs a B200 keeps resident
constexpr int kMaxDevices = 64;

// the CTA whose range holds entry e (ranges: [c*E/C, (c+1)*E/C))
__device__ __forceinline__ long long cta_of(long long e, long long E, long long C) {
  return ((e + 1) * C - 1) / E;
}

template <int NT>
__device__ int block_excl_scan(int v, int *tmp, int &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int nw = NT / 32;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += t;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? tmp[lane] : 0, incl = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane < nw) tmp[lane] = incl - w;
    if (lane == nw - 1) tmp[32] = incl;
  }
  __syncthreads();
  const int r = tmp[warp] + x - v;
  total = tmp[32];
  __syncthreads();
  return r;
}


constexpr int kNQ = 16;                 // MMA N: the heads of a group, zero padded
constexpr int kTile = 8192;             // 64 rows x 64 bf16, one swizzled tile
constexpr int kUnitBytes = 4 * kTile;   // K lo | V lo | K hi | V hi
constexpr int kMaxEnt = 128;            // list entries one CTA may own (one per thread)

struct TcArgs {
  const uint16_t *Q;
  uint16_t *O;
  const int32_t *idx;
  const int32_t *phys;  // SPARDA_ADDR_PHYS: the slot of each entry
  const int32_t *seq_len;  // optional per-sequence lengths (decode: nq = 1)
  float *ws_o;          // [pairs][max_cover][R][128] unnormalised segment outputs
  float2 *ws_ml;        // [pairs][max_cover][R] (max, sum) in the exp2 domain
  uint32_t *counters;   // [pairs] tickets, zero between calls
  int32_t *status;
  long long n_entries;  // pairs * S
  long long bg_rows, blk_rows;  // strides in 128-element rows
  int G, S, NB, addr_mode, nq, q_start, max_cover;
  int order_bgi;        // 1: pairs are streamed in (sequence, group, token) order
  int n_slots;          // SPARDA_ADDR_PHYS: slots per (sequence, group)
  int T;
  int split_kv;         // 1: a slot's K and V tiles are refilled separately (see the producer;
                        // picks the kernel instance, 2 or 3 stages)
  float scale_log2;
  long long wait_cycles;  // bound of every wait of the pipeline, in SM clock cycles
};

// Memory index (b * nq + i) * G + g of the pair at stream position p.  With
// several query tokens (prefill) the pairs are streamed group by group, so
// the CTAs running at one time read the K/V of one (sequence, group) --
// 64 MB at 128K tokens, which stays in L2 -- rather than of every group.
__device__ __forceinline__ long long mem_pair(const TcArgs &a, long long p) {
  if (!a.order_bgi) return p;
  const long long i = p % a.nq, t = p / a.nq;
  return ((t / a.G) * a.nq + i) * a.G + t % a.G;
}

// Everything else a CTA keeps in shared memory; it sits in the dynamic
// allocation behind the operands, so the kernel has no static shared memory
// and the allocation starts on the 1024-byte boundary the swizzled tiles need.
template <int NSTAGE, bool SPLIT>
struct TcCtl {
  uint64_t full_bar[NSTAGE], empty_bar[NSTAGE];    // a slot's K tiles: landed / read by S^T
  // with SPLIT, its V tiles: landed / read by O^T (else unused)
  uint64_t fullv_bar[SPLIT ? NSTAGE : 1], emptyv_bar[SPLIT ? NSTAGE : 1];
  uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
  uint32_t tmem_base;
  int s_last;
  int s_abort;
  int s_tmp[33];
  int s_row[kMaxEnt];   // TMA row coordinate of the block
  int s_rows[kMaxEnt];  // keys of the block at or before the query
  int s_seg[kMaxEnt];   // segment (pair - pair0)
  float red[2][kNQ];    // per-warp block maxima (softmax warps)
  float corr_s[2][kNQ]; // rescale factor of a block (double buffer)
  float seg_m[4][kNQ];  // running max at a segment's end (ring of 4)
  float seg_l[4][2][kNQ];  // per-warp sums at a segment's end
};

// stages | Q^T operand (16 rows x 128 dims) | two P^T operands | control
template <int NSTAGE, bool SPLIT>
constexpr size_t tc_smem() {
  return (size_t)NSTAGE * kUnitBytes + 4096 + 2 * 2048 +
         (sizeof(TcCtl<NSTAGE, SPLIT>) + 127) / 128 * 128;
}

constexpr int kWarps = 9;               // 4 correction, producer, 2 MMA issuers, 2 softmax warps
constexpr int kWsThreads = kWarps * 32;
constexpr int kBarSoftmax = 1;          // named barrier: the two softmax warps
constexpr int kBarCorr = 2;             // named barrier: the four correction warps
constexpr int kWarpProducer = 2, kWarpMma = 3, kWarpMma2 = 8;  // softmax: 4, 5; correction: 0, 1, 6, 7

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// barrier among n threads that also ORs a flag over them
__device__ __forceinline__ bool named_sync_or(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// bounded wait (limit in SM clock cycles) that also gives up when another
// role has given up
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag, long long limit) {
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

// Device-scope ticket with acquire-release ordering.
__device__ __forceinline__ unsigned ticket_acq_rel(uint32_t *p) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

// End of a segment, run by the 128 correction threads (thread = output
// dim): normalise and write the pair's output if this CTA covers the whole
// pair, else store the segment's (max, sum, unnormalised output) and let the
// last CTA to finish the pair combine them.
template <int R>
__device__ __forceinline__ void seg_flush(const TcArgs &a, long long pair, bool live, long long E,
                                          long long NC, const float (&acc)[R], const float *st_m,
                                          const float *st_l, int *s_last, int dim) {
  const long long c_first = cta_of(pair * a.S, E, NC);
  const long long c_last = cta_of(pair * a.S + a.S - 1, E, NC);
  const int n_cover = (int)(c_last - c_first + 1);
  const long long slot = pair * a.max_cover + (blockIdx.x - c_first);
#pragma unroll
  for (int h = 0; h < R; ++h) {
    const float L = live ? st_l[h] + st_l[kNQ + h] : 0.f;
    const float M = live ? st_m[h] : -INFINITY;
    const float o = live ? acc[h] : 0.f;
    if (n_cover == 1) {
      const float r = L > 0.f ? o / L : 0.f;
      a.O[(mem_pair(a, pair) * R + h) * kD + dim] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
    } else {
      a.ws_o[(slot * R + h) * kD + dim] = o;
      if (dim == 0) a.ws_ml[slot * R + h] = make_float2(M, L);
    }
  }
  if (n_cover > 1) {
    // the barrier orders every correction thread's stores before the ticket,
    // whose release publishes them device-wide; the last CTA's acquire (and
    // the barrier after it) orders its loads of the other segments after
    named_sync(kBarCorr, 128);
    if (dim == 0) *s_last = (ticket_acq_rel(&a.counters[pair]) == (unsigned)(n_cover - 1));
    named_sync(kBarCorr, 128);
    if (*s_last) {
      // merge the pair's segments online, up to four heads at a time, with
      // the loads of several segments in flight together
      const long long base = pair * a.max_cover;
      constexpr int HC = R < 4 ? R : 4;
      constexpr int NBAT = 8 / HC;
#pragma unroll 1
      for (int h0 = 0; h0 < R; h0 += HC) {
        float M[HC], L[HC], o[HC];
#pragma unroll
        for (int h = 0; h < HC; ++h) {
          M[h] = -INFINITY;
          L[h] = 0.f;
          o[h] = 0.f;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < n_cover; c0 += NBAT) {
          float2 ml[NBAT][HC];
          float ov[NBAT][HC];
#pragma unroll
          for (int q = 0; q < NBAT; ++q) {
#pragma unroll
            for (int h = 0; h < HC; ++h) {
              const bool in = c0 + q < n_cover;
              const long long sl = base + c0 + q;
              ml[q][h] = in ? __ldcg(&a.ws_ml[sl * R + h0 + h]) : make_float2(-INFINITY, 0.f);
              ov[q][h] = in ? __ldcg(&a.ws_o[(sl * R + h0 + h) * kD + dim]) : 0.f;
            }
          }
#pragma unroll
          for (int q = 0; q < NBAT; ++q) {
#pragma unroll
            for (int h = 0; h < HC; ++h) {
              if (ml[q][h].x == -INFINITY) continue;  // a segment with no keys, or none
              const float mn = fmaxf(M[h], ml[q][h].x);
              const float f_old = exp2f(M[h] - mn), f_new = exp2f(ml[q][h].x - mn);
              L[h] = L[h] * f_old + ml[q][h].y * f_new;
              o[h] = o[h] * f_old + ov[q][h] * f_new;
              M[h] = mn;
            }
          }
        }
#pragma unroll
        for (int h = 0; h < HC; ++h) {
          const float r = L[h] > 0.f ? o[h] / L[h] : 0.f;
          a.O[(mem_pair(a, pair) * R + h0 + h) * kD + dim] =
              __bfloat16_as_ushort(__float2bfloat16_rn(r));
        }
      }
      if (dim == 0) a.counters[pair] = 0u;
    }
  }
  named_sync(kBarCorr, 128);
}

// Two stages per CTA with three CTAs per SM keep as many blocks in flight as
// three stages with two CTAs, but give each SM three independent chains of
// (S^T, softmax, O^T): a stage is held from its landing until its O^T MMA is
// done, and more chains hide that hold better.  Sixteen heads per group need
// more registers than three CTAs per SM allow.
template <int R, int NSTAGE, bool SPLIT>
__global__ void __launch_bounds__(kWsThreads, (R <= 8 && NSTAGE <= 2) ? 3 : 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                   const __grid_constant__ TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = smem_raw;
  uint8_t *stages = sm;                          // NSTAGE x 32 KB
  uint8_t *qop = sm + NSTAGE * kUnitBytes;       // Q^T operand: 16 rows x 128 dims
  uint8_t *pop = qop + 4096;                     // two P^T operands: 16 rows x 64 keys
  TcCtl<NSTAGE, SPLIT> &ctl = *reinterpret_cast<TcCtl<NSTAGE, SPLIT> *>(pop + 2 * 2048);
  uint64_t *full_bar = ctl.full_bar, *empty_bar = ctl.empty_bar;
  uint64_t *fullv_bar = ctl.fullv_bar, *emptyv_bar = ctl.emptyv_bar;
  uint64_t *s_full = ctl.s_full, *p_full = ctl.p_full, *o_full = ctl.o_full, *o_free = ctl.o_free;
  int *s_row = ctl.s_row, *s_rows = ctl.s_rows, *s_seg = ctl.s_seg;
  volatile int *s_abort = &ctl.s_abort;
  float(*red)[kNQ] = ctl.red;
  float(*corr_s)[kNQ] = ctl.corr_s;
  float(*seg_m)[kNQ] = ctl.seg_m;
  float(*seg_l)[2][kNQ] = ctl.seg_l;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long lim = a.wait_cycles;
  const long long E = a.n_entries, NC = gridDim.x;
  const long long e0 = (long long)blockIdx.x * E / NC;
  const long long e1 = (long long)(blockIdx.x + 1) * E / NC;
  pdl_trigger();
  if (e0 >= e1) return;
  if (smem_addr(smem_raw) & 1023u) {  // the swizzled tiles would be misread
    pdl_wait();
    if (tid == 0) flag_status(a.status, SPARDA_DEV_LAYOUT);
    return;
  }
  const long long pair0 = e0 / a.S;
  const int n_seg = (int)((e1 - 1) / a.S - pair0 + 1);

  // barriers, TMEM and the zeroed operands are set up while the block list
  // is being loaded
  if (tid == 0) {
    for (int st = 0; st < NSTAGE; ++st) {
      mbar_init(&full_bar[st], 1);
      mbar_init(&empty_bar[st], 1);
      if (SPLIT) {
        mbar_init(&fullv_bar[st], 1);
        mbar_init(&emptyv_bar[st], 1);
      }
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 64);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_free[b], 128);
    }
    *s_abort = 0;
    fence_mbar_init();
    tc::prefetch_map(&mapK);
    tc::prefetch_map(&mapV);
  }
  pdl_wait();
  const long long e_me = e0 + tid;
  const long long pair_me = e_me / a.S;
  const int s_me = (int)(e_me - pair_me * a.S);
  const long long pm_me = mem_pair(a, pair_me);
  const bool own = tid < kMaxEnt && e_me < e1;
  const int j_me = own ? a.idx[pm_me * a.S + s_me] : -1;
  const int phys_me = (own && a.addr_mode == SPARDA_ADDR_PHYS) ? a.phys[pm_me * a.S + s_me] : 0;
  if (warp == 0) tc::tmem_alloc(&ctl.tmem_base, 64);
  for (int i = tid; i < (4096 + 4096) / 16; i += kWsThreads)  // Q^T, P^T rows >= R stay zero
    reinterpret_cast<uint4 *>(qop)[i] = make_uint4(0, 0, 0, 0);

  // ---- the range's valid entries, in order (at most kMaxEnt) ----
  int row_ = 0, rows_ = 0, seg_ = 0, cnt = 0;
  {
    const long long e = e_me;
    if (tid < kMaxEnt && e < e1) {
      const long long pair = pair_me, pm = pm_me;
      const int s = s_me;
      const int j = j_me;
      if (j >= 0) {
        int pos = a.q_start + (int)((pm / a.G) % a.nq);
        if (a.seq_len) {  // per-sequence lengths: the queries are the sequence's last nq tokens
          const int len = a.seq_len[(pm / a.G) / a.nq];
          pos = (len >= a.nq && len <= a.T) ? len - a.nq + (int)((pm / a.G) % a.nq)
                                            : -1;  // -1: every block is flagged
        }
        const bool slot_bad =
            a.addr_mode == SPARDA_ADDR_PHYS && (phys_me < 0 || phys_me >= a.n_slots);
        if (pos < 0 || j >= a.NB || j > pos / kBlk || slot_bad) {
          flag_status(a.status, SPARDA_DEV_RANGE);
        } else {
          const long long kvpair = (pm / a.G) / a.nq * a.G + pm % a.G;
          const int m = a.addr_mode == SPARDA_ADDR_SLOT ? s
                        : a.addr_mode == SPARDA_ADDR_PHYS ? phys_me
                                                          : j;
          row_ = (int)(kvpair * a.bg_rows + (long long)m * a.blk_rows);
          rows_ = min(kBlk, pos + 1 - j * kBlk);
          seg_ = (int)(pair - pair0);
          cnt = 1;
        }
      }
    }
  }
  int nb;
  const int off = block_excl_scan<kWsThreads>(cnt, ctl.s_tmp, nb);
  if (cnt) {
    s_row[off] = row_;
    s_rows[off] = rows_;
    s_seg[off] = seg_;
  }
  fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ctl.tmem_base;  // S0 | S1 | O0 | O1, 16 columns each
  auto first_of = [&](int u) { return u == 0 || s_seg[u - 1] != s_seg[u]; };
  auto last_of = [&](int u) { return u == nb - 1 || s_seg[u + 1] != s_seg[u]; };

  int produced_k = 0, produced_v = 0;  // producer: blocks whose K / V loads were issued
  int issued_s = 0, issued_o = 0;      // MMA issuers (lane 0): products committed

  if (warp == kWarpProducer) {
    // ================= producer =================
    // A block's K and V tiles have barriers of their own.  In the SPLIT
    // variant (TcArgs::split_kv picks it), K(u) goes out as soon as
    // S^T(u - NSTAGE) has read its slot's K tiles
    // and V(u) once O^T(u - NSTAGE) has read the V tiles: V is then issued
    // later than K and lands about when the softmax of its block is done,
    // so neither half waits long in its slot.  That pays when the blocks
    // come from L2 (the prefill's shared blocks, ~1 us away), where the
    // hold in the slot is a large part of a block's time; from HBM (decode,
    // ~4 us under load) it does not, and both halves go out together.
    if (lane == 0 && !SPLIT) {
#pragma unroll 1
      for (int u = 0; u < nb; ++u) {
        const int st = u % NSTAGE;
        // one barrier per slot: all four tiles land on full_bar, and O^T
        // (the last reader) frees the slot on empty_bar
        if (u >= NSTAGE &&
            !wait_or_abort(&empty_bar[st], (uint32_t)(((u / NSTAGE) - 1) & 1), s_abort, lim))
          break;
        uint8_t *dst = stages + st * kUnitBytes;
        const int row = s_row[u];
        mbar_arrive_expect_tx(&full_bar[st], kUnitBytes);
        tc::tma_load_2d(dst, &mapK, 0, row, &full_bar[st]);
        tc::tma_load_2d(dst + kTile, &mapV, 0, row, &full_bar[st]);
        tc::tma_load_2d(dst + 2 * kTile, &mapK, 64, row, &full_bar[st]);
        tc::tma_load_2d(dst + 3 * kTile, &mapV, 64, row, &full_bar[st]);
        produced_k = u + 1;
      }
    } else if (lane == 0) {
      int uk = 0, uv = 0;
      long long t0 = clock64();
#pragma unroll 1
      while (uv < nb) {
        bool moved = false;
        if (uk < nb &&
            (uk < NSTAGE ||
             mbar_test_wait(&empty_bar[uk % NSTAGE], (uint32_t)(((uk / NSTAGE) - 1) & 1)))) {
          const int st = uk % NSTAGE;
          uint8_t *dst = stages + st * kUnitBytes;
          const int row = s_row[uk];
          mbar_arrive_expect_tx(&full_bar[st], 2 * kTile);
          tc::tma_load_2d(dst, &mapK, 0, row, &full_bar[st]);
          tc::tma_load_2d(dst + 2 * kTile, &mapK, 64, row, &full_bar[st]);
          produced_k = ++uk;
          moved = true;
        }
        if (uv < uk &&
            (uv < NSTAGE ||
             mbar_test_wait(&emptyv_bar[uv % NSTAGE], (uint32_t)(((uv / NSTAGE) - 1) & 1)))) {
          const int st = uv % NSTAGE;
          uint8_t *dst = stages + st * kUnitBytes;
          const int row = s_row[uv];
          mbar_arrive_expect_tx(&fullv_bar[st], 2 * kTile);
          tc::tma_load_2d(dst + kTile, &mapV, 0, row, &fullv_bar[st]);
          tc::tma_load_2d(dst + 3 * kTile, &mapV, 64, row, &fullv_bar[st]);
          produced_v = ++uv;
          moved = true;
        }
        if (moved) {
          t0 = clock64();
          continue;
        }
        if (*s_abort) break;
        if (clock64() - t0 > lim) {
          *s_abort = 1;
          break;
        }
        __nanosleep(20);
      }
    }
  } else if (warp == kWarpMma) {
    // ================= S^T issuer =================
    // S^T(u) as soon as its block's K tiles have landed and the softmax of
    // u-2 is done with S[u & 1]; in the SPLIT variant its completion frees
    // the slot's K tiles.
    // The query rows of the next segment are loaded into registers one
    // segment ahead, so their global-load latency overlaps the current one.
    constexpr uint32_t id1 = tc::idesc_bf16(128, kNQ, false, false);
    const uint64_t dK = tc::sdesc(stages, 16, 1024);
    const uint64_t dQ = tc::sdesc(qop, 16, 1024);
    constexpr int QV = (R * 16 + 31) / 32;  // 16-byte pieces of the query rows per lane
    uint4 qn[QV];
    auto load_q = [&](int seg) {
      const uint4 *src = reinterpret_cast<const uint4 *>(a.Q + mem_pair(a, pair0 + seg) * R * kD);
#pragma unroll
      for (int j = 0; j < QV; ++j) {
        const int i = lane + 32 * j;
        qn[j] = i < R * 16 ? ldg_stream(src + i) : make_uint4(0, 0, 0, 0);
      }
    };
    if (nb > 0) load_q(s_seg[0]);
    bool ok = true;
#pragma unroll 1
    for (int u = 0; u < nb && ok; ++u) {
      const int st = u % NSTAGE;
      ok = wait_or_abort(&full_bar[st], (uint32_t)((u / NSTAGE) & 1), s_abort, lim);
      if (ok && u >= 2) ok = wait_or_abort(&p_full[u & 1], (uint32_t)(((u - 2) >> 1) & 1), s_abort, lim);
      const bool first = first_of(u);
      if (ok && first && u >= 1)  // the previous S^T must be done with the old query
        ok = wait_or_abort(&s_full[(u - 1) & 1], (uint32_t)(((u - 1) >> 1) & 1), s_abort, lim);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      if (first) {
#pragma unroll
        for (int j = 0; j < QV; ++j) {
          const int i = lane + 32 * j;
          if (i < R * 16) {
            const int h = i >> 4, c8 = i & 15;
            *reinterpret_cast<uint4 *>(qop + (c8 >> 3) * 2048 + tc::sw128_offset(h, (c8 & 7) * 8)) = qn[j];
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        tc::fence_after_sync();
        const uint64_t base = dK + (uint64_t)(st * (kUnitBytes >> 4));
#pragma unroll
        for (int k = 0; k < 8; ++k)
          tc::mma_bf16(tmem + (u & 1) * kNQ, base + (uint64_t)((k >> 2) * (2 * kTile >> 4) + (k & 3) * 2),
                       dQ + (uint64_t)((k >> 2) * 128 + (k & 3) * 2), id1, k > 0);
        tc::mma_commit(&s_full[u & 1]);
        if (SPLIT) tc::mma_commit(&empty_bar[st]);  // the slot's K tiles are read
        issued_s = u + 1;
      }
      __syncwarp();
      if (first) {  // the next segment's query rows, off the critical path
        int u2 = u + 1;
        while (u2 < nb && s_seg[u2] == s_seg[u]) ++u2;
        if (u2 < nb) load_q(s_seg[u2]);
      }
    }
    if (!ok) *s_abort = 1;
  } else if (warp == kWarpMma2) {
    // ================= O^T issuer =================
    // O^T(v) as soon as the softmax of v is done, its V tiles have landed and
    // the correction of v-2 has read O[v & 1]; its completion frees the
    // slot's V tiles (outside the SPLIT variant: the whole slot, whose S^T
    // finished before its softmax began).
    constexpr uint32_t id2 = tc::idesc_bf16(128, kNQ, true, false);
    const uint64_t dV = tc::sdesc(stages + kTile, 2 * kTile, 1024);
    const uint64_t dP = tc::sdesc(pop, 16, 1024);
    bool ok = true;
#pragma unroll 1
    for (int v = 0; v < nb && ok; ++v) {
      const int st = v % NSTAGE;
      ok = wait_or_abort(&p_full[v & 1], (uint32_t)((v >> 1) & 1), s_abort, lim);
      if (ok && v >= 2) ok = wait_or_abort(&o_free[v & 1], (uint32_t)(((v - 2) >> 1) & 1), s_abort, lim);
      if (ok && SPLIT) ok = wait_or_abort(&fullv_bar[st], (uint32_t)((v / NSTAGE) & 1), s_abort, lim);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      if (lane == 0) {
        tc::fence_after_sync();
        const uint64_t base = dV + (uint64_t)(st * (kUnitBytes >> 4));
        const uint64_t bp = dP + (uint64_t)((v & 1) * (2048 >> 4));
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc::mma_bf16(tmem + 2 * kNQ + (v & 1) * kNQ, base + (uint64_t)(k * 128), bp + (uint64_t)(k * 2),
                       id2, k > 0);
        tc::mma_commit(&o_full[v & 1]);
        tc::mma_commit(SPLIT ? &emptyv_bar[st] : &empty_bar[st]);  // V tiles (or the slot) read
        issued_o = v + 1;
      }
      __syncwarp();
    }
    if (!ok) *s_abort = 1;
  } else if (warp == 4 || warp == 5) {
    // ================= softmax (thread = key of the block) =================
    const uint32_t lane_sel = (uint32_t)((warp & 3) * 32) << 16;
    const int key = tid - 128;
    float m_run[R], l_t[R];
    int smx_k = -1;  // count of segments with blocks, for the statistics ring
    bool ok = true;
#pragma unroll 1
    for (int u = 0; u < nb; ++u) {
      const int b = u & 1;
      if (first_of(u)) {
        ++smx_k;
#pragma unroll
        for (int h = 0; h < R; ++h) {
          m_run[h] = -INFINITY;
          l_t[h] = 0.f;
        }
      }
      if (ok) ok = wait_or_abort(&s_full[b], (uint32_t)((u >> 1) & 1), s_abort, lim);
      // block u-2 is fully corrected: its P^T and corr slots are free
      if (ok && u >= 2) ok = wait_or_abort(&o_free[b], (uint32_t)(((u - 2) >> 1) & 1), s_abort, lim);
      tc::fence_after_sync();
      float x[R];
      {
        float sv[16];
        tc::tmem_ld16(tmem + b * kNQ + lane_sel, sv);
        const bool valid = key < s_rows[u];
#pragma unroll
        for (int h = 0; h < R; ++h) x[h] = valid ? sv[h] * a.scale_log2 : -INFINITY;
#pragma unroll
        for (int h = 0; h < R; ++h) {
          const float mx = warp_max_xor(x[h], 1, 32);
          if (lane == 0) red[warp - 4][h] = mx;
        }
      }
      if (named_sync_or(kBarSoftmax, 64, !ok)) {
        ok = false;
        break;
      }
      float cr[R];
#pragma unroll
      for (int h = 0; h < R; ++h) {
        const float mn = fmaxf(m_run[h], fmaxf(red[0][h], red[1][h]));
        cr[h] = (mn == -INFINITY) ? 1.f : exp2f(m_run[h] - mn);
        m_run[h] = mn;
      }
      uint8_t *pb = pop + b * 2048;
#pragma unroll
      for (int h = 0; h < R; ++h) {
        const float p = (x[h] == -INFINITY) ? 0.f : exp2f(x[h] - m_run[h]);
        const __nv_bfloat16 pv = __float2bfloat16_rn(p);
        *reinterpret_cast<__nv_bfloat16 *>(pb + tc::sw128_offset(h, key)) = pv;
        l_t[h] = l_t[h] * cr[h] + __bfloat162float(pv);
      }
#pragma unroll
      for (int h = 0; h < R; ++h)  // unrolled: no dynamic register index
        if (key == h) corr_s[b][h] = cr[h];
      if (last_of(u)) {  // publish the segment's statistics
#pragma unroll
        for (int h = 0; h < R; ++h) {
          const float ls = warp_sum_xor(l_t[h], 1, 32);
          if (lane == 0) seg_l[smx_k & 3][warp - 4][h] = ls;
        }
#pragma unroll
        for (int h = 0; h < R; ++h)
          if (key == h) seg_m[smx_k & 3][h] = m_run[h];
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(&p_full[b]);
      // both softmax warps finish the block before either reuses red[]
      named_sync(kBarSoftmax, 64);
    }
    if (!ok) *s_abort = 1;
  } else {
    // ============ correction (warps 0, 1, 6, 7; thread = output dim) ============
    const int q = warp & 3;  // TMEM lane quadrant
    const uint32_t lane_sel = (uint32_t)(q * 32) << 16;
    const int dim = q * 32 + lane;
    float acc[R];
#pragma unroll
    for (int h = 0; h < R; ++h) acc[h] = 0.f;
    int cur = -1, next_flush = 0;
    int live_k = -1;  // count of segments with blocks seen so far
    bool ok = true;
    // The statistics of a segment ending at block v-1 were published before
    // p_full(v-1), which correction(v-1) already waited for.
#pragma unroll 1
    for (int v = 0; v < nb; ++v) {
      const int seg = s_seg[v];
      if (seg != cur) {
        if (named_sync_or(kBarCorr, 128, !ok)) {
          ok = false;
          break;
        }
        for (int f = next_flush; f < seg; ++f)
          seg_flush<R>(a, pair0 + f, f == cur, E, NC, acc, seg_m[live_k & 3],
                       &seg_l[live_k & 3][0][0], &ctl.s_last, dim);
        next_flush = seg;
        cur = seg;
        ++live_k;
#pragma unroll
        for (int h = 0; h < R; ++h) acc[h] = 0.f;
      }
      if (ok) ok = wait_or_abort(&o_full[v & 1], (uint32_t)((v >> 1) & 1), s_abort, lim);
      if (ok) ok = wait_or_abort(&p_full[v & 1], (uint32_t)((v >> 1) & 1), s_abort, lim);
      // one vote for all four warps, so they always leave at the same barrier
      if (named_sync_or(kBarCorr, 128, !ok)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float ov[16];
      tc::tmem_ld16(tmem + 2 * kNQ + (v & 1) * kNQ + lane_sel, ov);
#pragma unroll
      for (int h = 0; h < R; ++h) acc[h] = acc[h] * corr_s[v & 1][h] + ov[h];
      tc::fence_before_sync();
      mbar_arrive(&o_free[v & 1]);
    }
    // all four warps agree before the last flushes (which use the barrier).
    // After a timeout the segments not flushed yet are handed in as empty:
    // every pair's ticket count still completes, so the last CTA to finish a
    // pair resets its ticket and the workspace stays valid for the next call
    // (the outputs of this one are flagged SPARDA_DEV_TIMEOUT)
    if (named_sync_or(kBarCorr, 128, !ok)) ok = false;
    for (int f = next_flush; f < n_seg; ++f)
      seg_flush<R>(a, pair0 + f, ok && f == cur, E, NC, acc, seg_m[live_k & 3],
                   &seg_l[live_k & 3][0][0], &ctl.s_last, dim);
    if (!ok) *s_abort = 1;
  }

  __syncthreads();
  if (*s_abort) {
    // something never completed: give what was issued a bounded chance to
    // land before the CTA's memory is released; the status word says why
    flag_status(a.status, SPARDA_DEV_TIMEOUT);
    if (warp == kWarpProducer && lane == 0) {
      for (int u = max(0, produced_k - NSTAGE); u < produced_k; ++u)
        (void)mbar_wait_bounded(&full_bar[u % NSTAGE], (uint32_t)((u / NSTAGE) & 1));
      for (int u = max(0, produced_v - NSTAGE); u < produced_v; ++u)
        (void)mbar_wait_bounded(&fullv_bar[u % NSTAGE], (uint32_t)((u / NSTAGE) & 1));
    }
    // products still running read the ring and write TMEM: wait for the last
    // one each issuer committed (its operands were in shared memory when it
    // was issued, so it completes)
    if (warp == kWarpMma && lane == 0 && issued_s > 0)
      (void)mbar_wait_bounded(&s_full[(issued_s - 1) & 1], (uint32_t)(((issued_s - 1) >> 1) & 1));
    if (warp == kWarpMma2 && lane == 0 && issued_o > 0)
      (void)mbar_wait_bounded(&o_full[(issued_o - 1) & 1], (uint32_t)(((issued_o - 1) >> 1) & 1));
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

template <int R, int NSTAGE, bool SPLIT>
cudaError_t launch_tc(const CUtensorMap &mk, const CUtensorMap &mv, const TcArgs &a,
                      long long grid_max, long long grid_min, int forced, cudaStream_t stream) {
  constexpr size_t smem = tc_smem<NSTAGE, SPLIT>();
  auto kern = attn_tc_kernel<R, NSTAGE, SPLIT>;
  // per device, once: shared-memory attributes and how many CTAs stay
  // resident (one wave: as many CTAs as the device keeps resident, never
  // more than the plan sized the workspace for, never fewer than the lists
  // need)
  struct Cached {
    void *ctx;
    int resident;
  };
  static Cached cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void *ctx = current_context();
  int &resident_dev = cache[dev].resident;
  if (resident_dev == 0 || cache[dev].ctx != ctx) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    // resident CTAs per SM from the shared-memory budget (each CTA also
    // holds its static shared memory and the per-block reservation) and
    // from the register file (allocated per warp in 256-register units)
    int n_sm = 148, per_sm = 0, reserved = 0, regs_sm = 65536;
    (void)cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    (void)cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    (void)cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    (void)cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
    cudaFuncAttributes fa;
    size_t stat = 4096;
    int regs = 128;
    if (cudaFuncGetAttributes(&fa, kern) == cudaSuccess) {
      stat = fa.sharedSizeBytes;
      regs = fa.numRegs;
    }
    (void)cudaGetLastError();
    int occ = per_sm > 0 ? (int)((size_t)per_sm / (smem + stat + (size_t)reserved)) : 1;
    const int warp_regs = (regs * 32 + 255) / 256 * 256;
    occ = std::min(occ, regs_sm / (warp_regs * kWarps));
    occ = std::max(1, std::min(occ, 3));
    resident_dev = occ * n_sm;
    cache[dev].ctx = ctx;
  }
  long long grid = resident_dev;
  if (forced > 0) grid = forced;
  grid = std::max(grid, grid_min);
  grid = std::min(grid, grid_max);
  const cudaError_t e = launch_pdl(kern, (unsigned)grid, kWsThreads, smem, stream, mk, mv, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

DecodePlan plan_gather(const sparda_params &p, long long pairs) {
  DecodePlan pl{};
  pl.S = p.k + p.n_init + p.n_local;
  const int R = p.G > 0 ? p.Hq / p.G : 1;
  const long long E = pairs * pl.S;
  // the workspace is sized for the largest grid a launch may use
  long long C = std::max<long long>(kGridMax, ceil_div_ll(E, kMaxEnt));
  const int forced = tuning(p).attn_ctas;
  if (forced > 0) C = std::max<long long>(C, forced);
  if (C > E) C = E;
  if (C < 1) C = 1;
  pl.n_cta = C;
  pl.n_cta_min = std::min<long long>(C, ceil_div_ll(E, kMaxEnt));
  const long long w_min = std::max<long long>(E / C, 1);
  pl.max_cover = (int)(ceil_div_ll(pl.S, w_min) + 1);
  const size_t parts = (size_t)pairs * pl.max_cover * R;
  size_t off = ((parts * kD * 4) + 255) & ~(size_t)255;  // outputs
  pl.ws_ml_off = off;
  off += ((parts * 8) + 255) & ~(size_t)255;              // (max, sum)
  pl.ws_ticket_off = off;
  pl.ws_ticket_bytes = (size_t)pairs * 4;
  off += (pl.ws_ticket_bytes + 255) & ~(size_t)255;       // tickets
  pl.ws_bytes = off;
  return pl;
}

DecodePlan plan_decode(const sparda_params &p) { return plan_gather(p, (long long)p.B * p.G); }

namespace {
// The arguments and tensor maps of one attention launch.
cudaError_t build_tc(const sparda_params &p, const DecodePlan &pl, int nq, int q_start,
                     const uint16_t *Q, const uint16_t *K, const uint16_t *V, long long bg_stride,
                     long long blk_stride, const int32_t *idx, int addr_mode, uint16_t *O, void *ws,
                     int32_t *dev_status, const int32_t *phys, int n_slots, TcArgs &a,
                     CUtensorMap &mk, CUtensorMap &mv) {
  const long long pairs = (long long)p.B * nq * p.G;
  const long long kv_pairs = (long long)p.B * p.G;
  const int NB = (p.T + kBlk - 1) / kBlk;
  const long long bg_rows = bg_stride / kD, blk_rows = blk_stride / kD;
  // rows each tensor map may touch: up to the last row of the last block the
  // strides can address, but never past the packed end of the buffer
  const long long m_max = addr_mode == SPARDA_ADDR_SLOT   ? pl.S - 1
                          : addr_mode == SPARDA_ADDR_PHYS ? n_slots - 1
                                                          : NB - 1;
  long long extent = (kv_pairs - 1) * bg_rows + m_max * blk_rows + kBlk;
  extent = std::min(extent, kv_pairs * bg_rows);
  if (extent >= (1LL << 31)) return cudaErrorInvalidValue;
  if (!tc::make_map_2d(&mk, K, kD, (uint64_t)extent, kD, 64, 64) ||
      !tc::make_map_2d(&mv, V, kD, (uint64_t)extent, kD, 64, 64))
    return cudaErrorNotSupported;
  a = TcArgs{};
  a.Q = Q;
  a.O = O;
  a.idx = idx;
  a.phys = phys;
  a.seq_len = p.seq_len;
  a.T = p.T;
  a.n_slots = n_slots;
  a.status = dev_status;
  a.n_entries = pairs * pl.S;
  a.bg_rows = bg_rows;
  a.blk_rows = blk_rows;
  a.G = p.G;
  a.S = pl.S;
  a.NB = NB;
  a.addr_mode = addr_mode;
  a.nq = nq;
  a.q_start = q_start;
  a.max_cover = pl.max_cover;
  a.order_bgi = nq > 1 ? 1 : 0;
  const sparda_tuning &tu = tuning(p);
  a.split_kv = tu.attn_split_kv != 0 ? (tu.attn_split_kv > 0 ? 1 : 0) : (nq > 1 ? 1 : 0);
  a.wait_cycles = tu.attn_wait_cycles > 0 ? tu.attn_wait_cycles : kWaitCycles;
  const float scale = p.scale > 0.f ? p.scale : 1.0f / sqrtf((float)p.d);
  a.scale_log2 = scale * kLog2e;
  char *w = static_cast<char *>(ws);
  a.ws_o = reinterpret_cast<float *>(w);
  a.ws_ml = reinterpret_cast<float2 *>(w + pl.ws_ml_off);
  a.counters = reinterpret_cast<uint32_t *>(w + pl.ws_ticket_off);
  return cudaSuccess;
}

// ring depth: 2 x 32 KB with three resident CTAs per SM where the registers
// allow it (up to 8 heads per group), else 3 x 32 KB with two; 4 and 6 (one
// CTA per SM) stay selectable through sparda_tuning
int ring_stages(const sparda_params &p) {
  const int R = p.Hq / p.G;
  const int st = tuning(p).attn_stages;
  return st != 0 ? st : (R <= 8 ? 2 : 3);
}
}  // namespace

cudaError_t launch_gather_attn(const sparda_params &p, const DecodePlan &pl, int nq, int q_start,
                               const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                               long long bg_stride, long long blk_stride, const int32_t *idx,
                               int addr_mode, uint16_t *O, void *ws, int32_t *dev_status,
                               cudaStream_t stream, const int32_t *phys, int n_slots) {
  if ((long long)p.B * nq * p.G == 0) return cudaSuccess;
  const int R = p.Hq / p.G;
  TcArgs a;
  CUtensorMap mk, mv;
  const cudaError_t eb = build_tc(p, pl, nq, q_start, Q, K, V, bg_stride, blk_stride, idx,
                                  addr_mode, O, ws, dev_status, phys, n_slots, a, mk, mv);
  if (eb != cudaSuccess) return eb;
  const sparda_tuning &tu = tuning(p);
  const int stages = ring_stages(p);
  const int fc = tu.attn_ctas;
#define SPARDA_LAUNCH_R(RR)                                                                    \
  if (a.split_kv && stages <= 2) return launch_tc<RR, 2, true>(mk, mv, a, pl.n_cta, pl.n_cta_min, fc, stream); \
  if (a.split_kv && stages == 3) return launch_tc<RR, 3, true>(mk, mv, a, pl.n_cta, pl.n_cta_min, fc, stream); \
  if (stages <= 2) return launch_tc<RR, 2, false>(mk, mv, a, pl.n_cta, pl.n_cta_min, fc, stream); \
  if (stages == 3) return launch_tc<RR, 3, false>(mk, mv, a, pl.n_cta, pl.n_cta_min, fc, stream); \
  if (stages == 4) return launch_tc<RR, 4, false>(mk, mv, a, pl.n_cta, pl.n_cta_min, fc, stream); \
  return launch_tc<RR, 6, false>(mk, mv, a, pl.n_cta, pl.n_cta_min, fc, stream);
  switch (R) {
    case 1: SPARDA_LAUNCH_R(1)
    case 2: SPARDA_LAUNCH_R(2)
    case 4: SPARDA_LAUNCH_R(4)
    case 8: SPARDA_LAUNCH_R(8)
    case 16: SPARDA_LAUNCH_R(16)
    default: return cudaErrorInvalidValue;
  }
#undef SPARDA_LAUNCH_R
}

cudaError_t launch_attn_decode(const sparda_params &p, const DecodePlan &pl, const uint16_t *Q,
                               const uint16_t *K, const uint16_t *V, long long bg_stride,
                               long long blk_stride, const int32_t *idx, int addr_mode,
                               uint16_t *O, void *ws, int32_t *dev_status, cudaStream_t stream,
                               const int32_t *phys, int n_slots) {
  return launch_gather_attn(p, pl, 1, p.T - 1, Q, K, V, bg_stride, blk_stride, idx, addr_mode, O,
                            ws, dev_status, stream, phys, n_slots);
}

}  // namespace sparda
