// attn_decode.cu -- GQA block-sparse attention of single query tokens over
// their own block lists (decode; also the per-token prefill path).
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
//    of two resident CTAs per SM -- one wave, no tail.  A range may start or
//    end inside a pair; each piece of a pair is a "segment";
//  - the entry list of a range is read by all threads at once and compacted
//    with a block scan (one global-load latency per CTA);
//  - TMA (cp.async.bulk.tensor, 128-byte swizzle, no multicast) stages each
//    block as [K lo-dims | V lo-dims | K hi-dims | V hi-dims] (8 KB each) in
//    an NSTAGE ring, with the pair's query rows at the first block of a
//    segment.  The M = 128 MMA for S^T reads rows 0-63 = the block's keys;
//    its rows 64-127 alias the finite V tiles and are masked;
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
constexpr int kThreads = 128;

struct TcArgs {
  const uint16_t *Q;
  uint16_t *O;
  const int32_t *idx;
  float *ws_o;          // [pairs][max_cover][R][128] unnormalised segment outputs
  float2 *ws_ml;        // [pairs][max_cover][R] (max, sum) in the exp2 domain
  uint32_t *counters;   // [pairs] tickets, zero between calls
  int32_t *status;
  long long n_entries;  // pairs * S
  long long bg_rows, blk_rows;  // strides in 128-element rows
  int G, S, NB, addr_mode, nq, q_start, max_cover;
  float scale_log2;
};

template <int R>
struct TcCfg {
  static constexpr int QB = R * kD * 2;  // raw query rows of one pair
  static constexpr int QB_AL = (QB + 127) / 128 * 128;
  // stages (1024-aligned) | raw query ring | Q^T operand | P^T operand | slack
  static size_t smem(int nstage) {
    return (size_t)nstage * kUnitBytes + (size_t)nstage * QB_AL + 4096 + 2048 + 1024;
  }
};

// End of a segment: normalise and write the pair's output if this CTA covers
// the whole pair, else store the segment's (max, sum, unnormalised output) and
// let the last CTA to finish the pair combine all of them.  Block-wide.
template <int R>
__device__ __forceinline__ void segment_flush(const TcArgs &a, long long pair, bool live,
                                              long long E, long long NC, const float (&acc)[R],
                                              const float (&m_run)[R], const float (&l_w)[R],
                                              float (*red)[kNQ], int *s_last) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (lane == 0)
#pragma unroll
    for (int h = 0; h < R; ++h) red[warp][h] = live ? l_w[h] : 0.f;
  __syncthreads();
  const long long c_first = cta_of(pair * a.S, E, NC);
  const long long c_last = cta_of(pair * a.S + a.S - 1, E, NC);
  const int n_cover = (int)(c_last - c_first + 1);
  const long long slot = pair * a.max_cover + (blockIdx.x - c_first);
  const int dim = tid;
#pragma unroll
  for (int h = 0; h < R; ++h) {
    const float L = red[0][h] + red[1][h] + red[2][h] + red[3][h];
    const float o = live ? acc[h] : 0.f;
    const float M = live ? m_run[h] : -INFINITY;
    if (n_cover == 1) {
      const float r = L > 0.f ? o / L : 0.f;
      a.O[(pair * R + h) * kD + dim] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
    } else {
      a.ws_o[(slot * R + h) * kD + dim] = o;
      if (dim == 0) a.ws_ml[slot * R + h] = make_float2(M, L);
    }
  }
  if (n_cover > 1) {
    __threadfence();
    __syncthreads();
    if (tid == 0) *s_last = (atomicAdd(&a.counters[pair], 1u) == (unsigned)(n_cover - 1));
    __syncthreads();
    if (*s_last) {
      __threadfence();
      const long long base = pair * a.max_cover;
#pragma unroll 1
      for (int h = 0; h < R; ++h) {
        float M = -INFINITY;
        for (int c = 0; c < n_cover; ++c) M = fmaxf(M, __ldcg(&a.ws_ml[(base + c) * R + h].x));
        float L = 0.f, o = 0.f;
        for (int c = 0; c < n_cover; ++c) {
          const float2 ml = __ldcg(&a.ws_ml[(base + c) * R + h]);
          const float fw = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
          L += fw * ml.y;
          o += fw * __ldcg(&a.ws_o[((base + c) * R + h) * kD + dim]);
        }
        const float r = L > 0.f ? o / L : 0.f;
        a.O[(pair * R + h) * kD + dim] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
      }
      if (tid == 0) a.counters[pair] = 0u;
    }
  }
  __syncthreads();
}

template <int R, int NSTAGE>
__global__ void __launch_bounds__(kThreads) attn_tc_kernel(const __grid_constant__ CUtensorMap mapK,
                                                           const __grid_constant__ CUtensorMap mapV,
                                                           TcArgs a) {
  using C = TcCfg<R>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint8_t *stages = sm;                              // NSTAGE x 32 KB
  uint8_t *qop = sm + NSTAGE * kUnitBytes;           // Q^T operand: 16 rows x 128 dims
  uint8_t *pop = qop + 4096;                         // P^T operand: 16 rows x 64 keys
  uint8_t *qraw = pop + 2048;                        // NSTAGE raw query slots
  __shared__ __align__(8) uint64_t full_bar[NSTAGE];
  __shared__ __align__(8) uint64_t mma1_bar, mma2_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int s_row[kMaxEnt];   // TMA row coordinate of the block
  __shared__ int s_rows[kMaxEnt];  // keys of the block at or before the query
  __shared__ int s_seg[kMaxEnt];   // segment (pair - pair0)
  __shared__ int s_tmp[33];
  __shared__ int s_last;
  __shared__ float red[4][kNQ];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long E = a.n_entries, NC = gridDim.x;
  const long long e0 = (long long)blockIdx.x * E / NC;
  const long long e1 = (long long)(blockIdx.x + 1) * E / NC;
  if (e0 >= e1) return;
  const long long pair0 = e0 / a.S;
  const int n_seg = (int)((e1 - 1) / a.S - pair0 + 1);

  // ---- the range's valid entries, in order (at most kMaxEnt) ----
  int row_ = 0, rows_ = 0, seg_ = 0, cnt = 0;
  {
    const long long e = e0 + tid;
    if (tid < kMaxEnt && e < e1) {
      const long long pair = e / a.S;
      const int s = (int)(e - pair * a.S);
      const int j = a.idx[e];
      if (j >= 0) {
        const int pos = a.q_start + (int)((pair / a.G) % a.nq);
        if (j >= a.NB || j > pos / kBlk) {
          flag_status(a.status, SPARDA_DEV_RANGE);
        } else {
          const long long kvpair = (pair / a.G) / a.nq * a.G + pair % a.G;
          const int m = a.addr_mode == SPARDA_ADDR_SLOT ? s : j;
          row_ = (int)(kvpair * a.bg_rows + (long long)m * a.blk_rows);
          rows_ = min(kBlk, pos + 1 - j * kBlk);
          seg_ = (int)(pair - pair0);
          cnt = 1;
        }
      }
    }
  }
  int nb;
  const int off = block_excl_scan<kThreads>(cnt, s_tmp, nb);
  if (cnt) {
    s_row[off] = row_;
    s_rows[off] = rows_;
    s_seg[off] = seg_;
  }
  if (tid == 0) {
    for (int st = 0; st < NSTAGE; ++st) mbar_init(&full_bar[st], 1);
    mbar_init(&mma1_bar, 1);
    mbar_init(&mma2_bar, 1);
    fence_mbar_init();
    tc::prefetch_map(&mapK);
    tc::prefetch_map(&mapV);
  }
  if (warp == 0) tc::tmem_alloc(&tmem_base, 32);
  // operand tiles start zeroed: rows >= R of Q^T and P^T stay zero
  for (int i = tid; i < (4096 + 2048) / 16; i += kThreads)
    reinterpret_cast<uint4 *>(qop)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base;
  const uint32_t tS = tmem, tO = tmem + kNQ;
  const uint32_t lane_sel = (uint32_t)(warp * 32) << 16;
  constexpr uint32_t id1 = tc::idesc_bf16(128, kNQ, false, false);
  constexpr uint32_t id2 = tc::idesc_bf16(128, kNQ, true, false);
  // operand descriptors: fixed bases, advanced in 16-byte units
  const uint64_t dK = tc::sdesc(stages, 16, 1024);          // S^T A operand (K tiles)
  const uint64_t dV = tc::sdesc(stages + kTile, 2 * kTile, 1024);  // O^T A operand (V^T)
  const uint64_t dQ = tc::sdesc(qop, 16, 1024);
  const uint64_t dP = tc::sdesc(pop, 16, 1024);

  // thread 0 only: TMA for block bi into its stage (+ the pair's query rows
  // at the first block of a segment)
  auto issue = [&](int bi) {
    const int st = bi % NSTAGE;
    const int seg = s_seg[bi];
    const bool first = bi == 0 || s_seg[bi - 1] != seg;
    uint8_t *dst = stages + st * kUnitBytes;
    const int row = s_row[bi];
    mbar_arrive_expect_tx(&full_bar[st], kUnitBytes + (first ? C::QB : 0));
    tc::tma_load_2d(dst, &mapK, 0, row, &full_bar[st]);
    tc::tma_load_2d(dst + kTile, &mapV, 0, row, &full_bar[st]);
    tc::tma_load_2d(dst + 2 * kTile, &mapK, 64, row, &full_bar[st]);
    tc::tma_load_2d(dst + 3 * kTile, &mapV, 64, row, &full_bar[st]);
    if (first) bulk_g2s(qraw + st * C::QB_AL, a.Q + (pair0 + seg) * R * kD, C::QB, &full_bar[st]);
  };
  // thread 0 only: S^T = K Q^T for block bi (rows 0-63 are its keys)
  auto mma1 = [&](int bi) {
    const uint64_t base = dK + (uint64_t)((bi % NSTAGE) * (kUnitBytes >> 4));
    tc::fence_after_sync();
#pragma unroll
    for (int k = 0; k < 8; ++k)
      tc::mma_bf16(tS, base + (uint64_t)((k >> 2) * (2 * kTile >> 4) + (k & 3) * 2),
                   dQ + (uint64_t)((k >> 2) * 128 + (k & 3) * 2), id1, k > 0);
    tc::mma_commit(&mma1_bar);
  };
  if (tid == 0)
    for (int bi = 0; bi < min(nb, NSTAGE); ++bi) issue(bi);

  // per thread: acc = one output dim (tid) of every head; m_run uniform;
  // l_w = this warp's share of the probability sums
  float acc[R], m_run[R], l_w[R];
#pragma unroll
  for (int h = 0; h < R; ++h) {
    acc[h] = 0.f;
    m_run[h] = -INFINITY;
    l_w[h] = 0.f;
  }
  uint32_t ph1 = 0, ph2 = 0;
  int early = -1;        // thread 0: block whose MMA1 is already in flight
  bool bad = false;      // this thread saw a wait give up
  int cur = -1, next_flush = 0, abort_at = -1;
  int issued_to = min(nb, NSTAGE);  // thread 0: blocks [0, issued_to) have TMA issued

#pragma unroll 1
  for (int bi = 0; bi < nb; ++bi) {
    const int st = bi % NSTAGE;
    const uint32_t tph = (uint32_t)((bi / NSTAGE) & 1);
    const int seg = s_seg[bi];
    if (seg != cur) {  // a new segment: its query arrived with this block
      for (int f = next_flush; f < seg; ++f)
        segment_flush<R>(a, pair0 + f, f == cur, E, NC, acc, m_run, l_w, red, &s_last);
      next_flush = seg;
      cur = seg;
#pragma unroll
      for (int h = 0; h < R; ++h) {
        acc[h] = 0.f;
        m_run[h] = -INFINITY;
        l_w[h] = 0.f;
      }
      if (!mbar_wait_bounded(&full_bar[st], tph)) bad = true;
      if (__syncthreads_or(bad)) {
        abort_at = bi;
        break;
      }
      const uint4 *q = reinterpret_cast<const uint4 *>(qraw + st * C::QB_AL);
      for (int i = tid; i < R * 16; i += kThreads) {
        const int h = i >> 4, c8 = i & 15;
        *reinterpret_cast<uint4 *>(qop + (c8 >> 3) * 2048 + tc::sw128_offset(h, (c8 & 7) * 8)) = q[i];
      }
      fence_proxy_async_smem();
      __syncthreads();
    }
    if (tid == 0 && early != bi) {
      if (mbar_wait_bounded(&full_bar[st], tph)) mma1(bi);
      else bad = true;
    }
    if (!mbar_wait_bounded(&mma1_bar, ph1)) bad = true;
    ph1 ^= 1;
    tc::fence_after_sync();

    // ---- softmax over this block's keys (thread = key, in warps 0 and 1) ----
    const int rows = s_rows[bi];
    float x[R];
    if (warp < 2) {
      float sv[16];
      tc::tmem_ld16(tS + lane_sel, sv);
      const bool valid = tid < rows;
#pragma unroll
      for (int h = 0; h < R; ++h) x[h] = valid ? sv[h] * a.scale_log2 : -INFINITY;
#pragma unroll
      for (int h = 0; h < R; ++h) {
        const float mx = warp_max_xor(x[h], 1, 32);
        if (lane == 0) red[warp][h] = mx;
      }
    }
    tc::fence_before_sync();
    if (__syncthreads_or(bad)) {
      abort_at = bi;
      break;
    }
    float corr[R];
#pragma unroll
    for (int h = 0; h < R; ++h) {
      const float mn = fmaxf(m_run[h], fmaxf(red[0][h], red[1][h]));
      corr[h] = (mn == -INFINITY) ? 1.f : exp2f(m_run[h] - mn);
      m_run[h] = mn;
      l_w[h] *= corr[h];
    }
    float pr[R];
    if (warp < 2) {
#pragma unroll
      for (int h = 0; h < R; ++h) {
        const float p = (x[h] == -INFINITY) ? 0.f : exp2f(x[h] - m_run[h]);
        const __nv_bfloat16 pb = __float2bfloat16_rn(p);
        *reinterpret_cast<__nv_bfloat16 *>(pop + tc::sw128_offset(h, tid)) = pb;
        pr[h] = __bfloat162float(pb);
      }
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();

    // ---- O^T(block) = V^T P^T; the next block's S^T right behind it ----
    if (tid == 0) {
      tc::fence_after_sync();
      const uint64_t base = dV + (uint64_t)(st * (kUnitBytes >> 4));
#pragma unroll
      for (int k = 0; k < 4; ++k)
        tc::mma_bf16(tO, base + (uint64_t)(k * 128), dP + (uint64_t)(k * 2), id2, k > 0);
      tc::mma_commit(&mma2_bar);
      const int nx = bi + 1;
      if (nx < nb && s_seg[nx] == seg &&
          mbar_test_wait(&full_bar[nx % NSTAGE], (uint32_t)((nx / NSTAGE) & 1))) {
        mma1(nx);
        early = nx;
      }
    }
    if (warp < 2) {  // probability sums, while the tensor core works
#pragma unroll
      for (int h = 0; h < R; ++h) l_w[h] += warp_sum_xor(pr[h], 1, 32);
    }
    if (!mbar_wait_bounded(&mma2_bar, ph2)) bad = true;
    ph2 ^= 1;
    tc::fence_after_sync();
    // both MMAs of block bi are done: its stage can be refilled
    if (tid == 0 && bi + NSTAGE < nb && !bad) {
      issue(bi + NSTAGE);
      issued_to = bi + NSTAGE + 1;
    }
    {
      float ov[16];
      tc::tmem_ld16(tO + lane_sel, ov);
#pragma unroll
      for (int h = 0; h < R; ++h) acc[h] = acc[h] * corr[h] + ov[h];
    }
    tc::fence_before_sync();
  }
  if (abort_at < 0 && __syncthreads_or(bad)) abort_at = nb;

  if (abort_at >= 0) {
    // something never completed: let what was issued land (bounded), then
    // free TMEM and leave; the status word says why
    flag_status(a.status, SPARDA_DEV_TIMEOUT);
    if (tid == 0) {
      for (int bj = max(0, abort_at); bj < issued_to; ++bj)
        (void)mbar_wait_bounded(&full_bar[bj % NSTAGE], (uint32_t)((bj / NSTAGE) & 1));
      (void)mbar_wait_bounded(&mma1_bar, ph1);
      (void)mbar_wait_bounded(&mma2_bar, ph2);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 32);
    return;
  }
  for (int f = next_flush; f < n_seg; ++f)
    segment_flush<R>(a, pair0 + f, f == cur, E, NC, acc, m_run, l_w, red, &s_last);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 32);
}

template <int R, int NSTAGE>
cudaError_t launch_tc(const CUtensorMap &mk, const CUtensorMap &mv, const TcArgs &a,
                      long long grid_max, long long grid_min, cudaStream_t stream) {
  const size_t smem = TcCfg<R>::smem(NSTAGE);
  auto kern = attn_tc_kernel<R, NSTAGE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // one wave: as many CTAs as the device keeps resident (never more than
  // the plan sized the workspace for, never fewer than the lists need)
  int dev = 0, n_sm = 148, occ = 1;
  if (cudaGetDevice(&dev) == cudaSuccess)
    (void)cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, smem) != cudaSuccess || occ < 1)
    occ = 1;
  (void)cudaGetLastError();
  long long grid = (long long)occ * n_sm;
  const int forced = env_int("SPARDA_DECODE_CTAS");
  if (forced > 0) grid = forced;
  grid = std::max(grid, grid_min);
  grid = std::min(grid, grid_max);
  kern<<<(unsigned)grid, kThreads, smem, stream>>>(mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

DecodePlan plan_gather(const sparda_params &p, long long pairs) {
  DecodePlan pl{};
  pl.S = p.k + p.n_init + p.n_local;
  const int R = p.G > 0 ? p.Hq / p.G : 1;
  const long long E = pairs * pl.S;
  // the workspace is sized for the largest grid a launch may use
  long long C = std::max<long long>(kGridMax, ceil_div_ll(E, kMaxEnt));
  const int forced = env_int("SPARDA_DECODE_CTAS");
  if (forced > 0) C = std::max<long long>(C, forced);
  if (C > E) C = E;
  if (C < 1) C = 1;
  pl.n_cta = C;
  pl.n_cta_min = std::min<long long>(C, ceil_div_ll(E, kMaxEnt));
  const long long w_min = std::max<long long>(E / C, 1);
  pl.max_cover = (int)(ceil_div_ll(pl.S, w_min) + 1);
  const size_t parts = (size_t)pairs * pl.max_cover * R;
  size_t off = ((parts * kD * 4) + 255) & ~(size_t)255;  // outputs
  off += ((parts * 8) + 255) & ~(size_t)255;              // (max, sum)
  off += (((size_t)pairs * 4) + 255) & ~(size_t)255;      // tickets
  pl.ws_bytes = off;
  return pl;
}

DecodePlan plan_decode(const sparda_params &p) { return plan_gather(p, (long long)p.B * p.G); }

cudaError_t launch_gather_attn(const sparda_params &p, const DecodePlan &pl, int nq, int q_start,
                               const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                               long long bg_stride, long long blk_stride, const int32_t *idx,
                               int addr_mode, uint16_t *O, void *ws, int32_t *dev_status,
                               cudaStream_t stream) {
  const long long pairs = (long long)p.B * nq * p.G;
  if (pairs == 0) return cudaSuccess;
  const int R = p.Hq / p.G;
  const long long kv_pairs = (long long)p.B * p.G;
  const int NB = (p.T + kBlk - 1) / kBlk;
  const long long bg_rows = bg_stride / kD, blk_rows = blk_stride / kD;
  // rows each tensor map may touch: up to the last row of the last block the
  // strides can address, but never past the packed end of the buffer
  const long long m_max = addr_mode == SPARDA_ADDR_SLOT ? pl.S - 1 : NB - 1;
  long long extent = (kv_pairs - 1) * bg_rows + m_max * blk_rows + kBlk;
  extent = std::min(extent, kv_pairs * bg_rows);
  if (extent >= (1LL << 31)) return cudaErrorInvalidValue;
  CUtensorMap mk, mv;
  if (!tc::make_map_2d(&mk, K, kD, (uint64_t)extent, kD, 64, 64) ||
      !tc::make_map_2d(&mv, V, kD, (uint64_t)extent, kD, 64, 64))
    return cudaErrorNotSupported;
  TcArgs a;
  a.Q = Q;
  a.O = O;
  a.idx = idx;
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
  const float scale = p.scale > 0.f ? p.scale : 1.0f / sqrtf((float)p.d);
  a.scale_log2 = scale * kLog2e;
  const size_t parts = (size_t)pairs * pl.max_cover * R;
  char *w = static_cast<char *>(ws);
  a.ws_o = reinterpret_cast<float *>(w);
  w += ((parts * kD * 4) + 255) & ~(size_t)255;
  a.ws_ml = reinterpret_cast<float2 *>(w);
  w += ((parts * 8) + 255) & ~(size_t)255;
  a.counters = reinterpret_cast<uint32_t *>(w);
  switch (R) {
    case 1: return launch_tc<1, 2>(mk, mv, a, pl.n_cta, pl.n_cta_min, stream);
    case 2: return launch_tc<2, 2>(mk, mv, a, pl.n_cta, pl.n_cta_min, stream);
    case 4: return launch_tc<4, 2>(mk, mv, a, pl.n_cta, pl.n_cta_min, stream);
    case 8: return launch_tc<8, 2>(mk, mv, a, pl.n_cta, pl.n_cta_min, stream);
    case 16: return launch_tc<16, 2>(mk, mv, a, pl.n_cta, pl.n_cta_min, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_decode(const sparda_params &p, const DecodePlan &pl, const uint16_t *Q,
                               const uint16_t *K, const uint16_t *V, long long bg_stride,
                               long long blk_stride, const int32_t *idx, int addr_mode,
                               uint16_t *O, void *ws, int32_t *dev_status, cudaStream_t stream) {
  return launch_gather_attn(p, pl, 1, p.T - 1, Q, K, V, bg_stride, blk_stride, idx, addr_mode, O,
                            ws, dev_status, stream);
}

}  // namespace sparda
