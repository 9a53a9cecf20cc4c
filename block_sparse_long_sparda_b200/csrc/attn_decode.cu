// attn_decode.cu -- GQA block-sparse attention of single query tokens over
// their own block lists (decode; also the per-token prefill path).
//
// [p4 "The fourth projection", Eq. 5 / Algorithm 2]: O_l = attention(Q_l,
// K_l[B_l], V_l[B_l]): each query head attends over the keys of its GQA
// group's selected blocks only; fp32 softmax and accumulation.
//
// Design (B200).  Decode attention reads 32 KB of K+V per selected block and
// does 2*R*128 fp32 FMA per key (the R query heads of a group share every
// key): about 4 FLOP/byte for R = 4, firmly HBM bound.  CUDA cores do the
// math; the work is organised to keep HBM busy from the first to the last
// microsecond:
//  - stream-K: the (query, group) "pairs" and their list entries are
//    flattened and cut into equal contiguous ranges, one per CTA, with a grid
//    of exactly two resident CTAs per SM -- one wave, no tail.  A range may
//    start or end inside a pair; each piece of a pair is a "segment";
//  - the entry list of the range is read by all threads at once and compacted
//    with a block scan (one global-load latency per CTA);
//  - every selected block (its K and V halves, plus the pair's query at the
//    first block of a segment) is staged by the bulk-copy engine
//    (cp.async.bulk, completion on an mbarrier) into an NSTAGE-deep ring that
//    runs across segment boundaries;
//  - the 64 keys of a staged block are split over the warps; within a warp,
//    QK^T keeps each lane's slice of the R query vectors in registers, every
//    lane converts only its own K elements, and a butterfly transpose-reduce
//    turns per-lane partials into whole dot products with one shuffle per
//    (key, head) pair; online softmax in the exp2 domain; P goes through a
//    small shared tile; PV with each lane owning 4 output dims of all R heads;
//  - at the end of a segment the warps merge in shared memory; a pair that a
//    single CTA covers is normalised and written at once, otherwise the
//    segment's (max, sum, unnormalised output) goes to the workspace and the
//    last CTA to finish the pair (atomic ticket, no waiting) combines them.
// Waits on the mbarriers are bounded: a timeout sets SPARDA_DEV_TIMEOUT, the
// CTA drains its copies (bounded) and leaves.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sparda {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kStageBytes = 2 * kBlk * kD * 2;  // K + V of one block = 32 KB
constexpr int kGridTarget = 2 * 148;            // two resident CTAs per B200 SM

struct DecArgs {
  const uint16_t *Q, *K, *V;
  long long bg_stride, blk_stride;
  const int32_t *idx;
  uint16_t *O;
  float *ws_o;          // [pairs][max_cover][R][128] unnormalised segment outputs
  float2 *ws_ml;        // [pairs][max_cover][R] (max, sum) in the exp2 domain
  uint32_t *counters;   // [pairs] tickets, zero between calls
  int32_t *status;
  long long n_entries;  // pairs * S
  int G, S, NB, addr_mode, nq, q_start, max_cover;
  float scale_log2;
};

template <int N>
__device__ __forceinline__ float transpose_reduce(float (&v)[N], int li) {
#pragma unroll
  for (int half = N / 2; half >= 1; half >>= 1) {
    const bool up = (li & half) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = up ? v[i] : v[i + half];
      const float keep = up ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
    }
  }
  return v[0];
}

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

template <int R, int NWARP>
struct Cfg {
  static constexpr int NT = NWARP * 32;
  static constexpr int DS = 64 / R;          // q dims per lane in QK
  static constexpr int LPK = 2 * R;          // lanes per key in QK
  static constexpr int KG = 32 / LPK;        // key groups per warp
  static constexpr int KW = kBlk / NWARP;    // keys per warp per block
  static constexpr int KPR = 2 * KG;         // keys per warp per QK round
  static constexpr int ROUNDS = KW / KPR;
  static constexpr int QBYTES = R * kD * 2;
  static constexpr int STAGE = kStageBytes + ((QBYTES + 127) / 128) * 128;
  static constexpr int MAX_ENT = 2 * NT;     // list entries one CTA may own
  // per-warp P tiles, rounded to 128 B so the warp-merge area after them
  // keeps the 16-byte alignment its vector stores need
  static constexpr int PBUF = (NWARP * (KW * R + R) + 31) / 32 * 32;
  static_assert(PBUF % 4 == 0, "merge area must stay 16-byte aligned");
  static size_t smem(int nstage) {
    return (size_t)nstage * STAGE + (size_t)PBUF * 4 + (size_t)NWARP * R * kD * 4 +
           (size_t)2 * NWARP * R * 4;
  }
};

template <int R, int NWARP, int NSTAGE>
__global__ void __launch_bounds__(NWARP * 32) attn_streamk_kernel(DecArgs a) {
  using C = Cfg<R, NWARP>;
  constexpr int NT = C::NT, DS = C::DS, LPK = C::LPK, KG = C::KG, KW = C::KW, KPR = C::KPR;
  constexpr int ROUNDS = C::ROUNDS;
  static_assert(ROUNDS >= 1 && KW % KPR == 0, "bad warp split");
  static_assert(DS >= 4, "R too large");

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *stages = smem;
  float *pbuf = reinterpret_cast<float *>(smem + NSTAGE * C::STAGE);
  float *red_o = pbuf + C::PBUF;                 // [NWARP][R][128]
  float *red_m = red_o + NWARP * R * kD;         // [NWARP][R]
  float *red_l = red_m + NWARP * R;              // [NWARP][R]
  __shared__ __align__(8) uint64_t full_bar[NSTAGE];
  __shared__ int s_m[C::MAX_ENT];
  __shared__ int s_rows[C::MAX_ENT];
  __shared__ int s_seg[C::MAX_ENT];
  __shared__ int s_tmp[33];
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long E = a.n_entries, NC = gridDim.x;
  const long long e0 = (long long)blockIdx.x * E / NC;
  const long long e1 = (long long)(blockIdx.x + 1) * E / NC;
  if (e0 >= e1) return;
  const long long pair0 = e0 / a.S;
  const int n_seg = (int)((e1 - 1) / a.S - pair0 + 1);

  // ---- the range's valid entries, in order ----
  int m_[2], rows_[2], seg_[2], cnt = 0;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const long long e = e0 + 2 * tid + u;
    if (e >= e1) continue;
    const long long pair = e / a.S;
    const int s = (int)(e - pair * a.S);
    const int j = a.idx[e];
    if (j < 0) continue;
    const int pos = a.q_start + (int)((pair / a.G) % a.nq);
    if (j >= a.NB || j > pos / kBlk) {
      flag_status(a.status, SPARDA_DEV_RANGE);
      continue;
    }
    m_[cnt] = a.addr_mode == SPARDA_ADDR_SLOT ? s : j;
    rows_[cnt] = min(kBlk, pos + 1 - j * kBlk);
    seg_[cnt] = (int)(pair - pair0);
    ++cnt;
  }
  int nb;
  const int off = block_excl_scan<NT>(cnt, s_tmp, nb);
  for (int u = 0; u < cnt; ++u) {
    s_m[off + u] = m_[u];
    s_rows[off + u] = rows_[u];
    s_seg[off + u] = seg_[u];
  }
  if (tid == 0) {
    for (int st = 0; st < NSTAGE; ++st) mbar_init(&full_bar[st], 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](int bi) {
    const int st = bi % NSTAGE;
    const int seg = s_seg[bi];
    const long long pair = pair0 + seg;
    const long long kvpair = (pair / a.G) / a.nq * a.G + pair % a.G;
    const uint32_t bytes = (uint32_t)s_rows[bi] * kD * 2;
    const bool first = bi == 0 || s_seg[bi - 1] != seg;
    uint8_t *dst = stages + st * C::STAGE;
    const long long off_kv = kvpair * a.bg_stride + (long long)s_m[bi] * a.blk_stride;
    mbar_arrive_expect_tx(&full_bar[st], 2 * bytes + (first ? C::QBYTES : 0));
    bulk_g2s(dst, a.K + off_kv, bytes, &full_bar[st]);
    bulk_g2s(dst + kStageBytes / 2, a.V + off_kv, bytes, &full_bar[st]);
    if (first) bulk_g2s(dst + kStageBytes, a.Q + pair * R * kD, C::QBYTES, &full_bar[st]);
  };
  if (tid == 0)
    for (int bi = 0; bi < min(nb, NSTAGE); ++bi) issue(bi);

  const int kg = lane / LPK, li = lane % LPK;
  const int my_head = li % R, my_kappa = li / R;
  float qv[R][DS];
  float m_run = -INFINITY, l_run = 0.f;  // for head my_head
  float acc[R][4];
#pragma unroll
  for (int h = 0; h < R; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
  float *pw = pbuf + warp * (KW * R + R);
  float *alpha = pw + KW * R;

  // ---- end of a segment: merge the warps, write or hand over ----
  auto flush = [&](int f, bool live) {
    const long long pair = pair0 + f;
#pragma unroll
    for (int h = 0; h < R; ++h)
      *reinterpret_cast<float4 *>(red_o + (warp * R + h) * kD + lane * 4) =
          live ? make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3])
               : make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane < R) {
      red_m[warp * R + lane] = live ? m_run : -INFINITY;
      red_l[warp * R + lane] = live ? l_run : 0.f;
    }
    __syncthreads();
    const long long c_first = cta_of(pair * a.S, E, NC);
    const long long c_last = cta_of(pair * a.S + a.S - 1, E, NC);
    const int n_cover = (int)(c_last - c_first + 1);
    const long long slot = pair * a.max_cover + (blockIdx.x - c_first);
    for (int t = tid; t < R * kD; t += NT) {
      const int h = t / kD, dim = t % kD;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NWARP; ++w) M = fmaxf(M, red_m[w * R + h]);
      float L = 0.f, o = 0.f;
#pragma unroll
      for (int w = 0; w < NWARP; ++w) {
        const float mw = red_m[w * R + h];
        const float fw = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        L += fw * red_l[w * R + h];
        o += fw * red_o[(w * R + h) * kD + dim];
      }
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
      if (tid == 0) s_last = (atomicAdd(&a.counters[pair], 1u) == (unsigned)(n_cover - 1));
      __syncthreads();
      if (s_last) {
        __threadfence();
        const long long base = pair * a.max_cover;
        for (int t = tid; t < R * kD; t += NT) {
          const int h = t / kD, dim = t % kD;
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
  };

  int cur = -1, next_flush = 0, abort_at = -1;
#pragma unroll 1
  for (int bi = 0; bi < nb; ++bi) {
    const int st = bi % NSTAGE;
    const bool ok = mbar_wait_bounded(&full_bar[st], (uint32_t)((bi / NSTAGE) & 1));
    if (!ok) flag_status(a.status, SPARDA_DEV_TIMEOUT);
    if (__syncthreads_or(!ok)) {
      abort_at = bi;
      break;
    }
    const uint8_t *stage = stages + st * C::STAGE;
    const int seg = s_seg[bi];
    if (seg != cur) {
      for (int f = next_flush; f < seg; ++f) flush(f, f == cur);
      next_flush = seg;
      cur = seg;
      m_run = -INFINITY;
      l_run = 0.f;
#pragma unroll
      for (int h = 0; h < R; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
      const uint16_t *qs = reinterpret_cast<const uint16_t *>(stage + kStageBytes);
#pragma unroll
      for (int h = 0; h < R; ++h) {
        if constexpr (DS >= 8) {
#pragma unroll
          for (int q8 = 0; q8 < DS / 8; ++q8) {
            const uint4 w = *reinterpret_cast<const uint4 *>(qs + h * kD + (q8 * LPK + li) * 8);
            qv[h][q8 * 8 + 0] = bf16_lo(w.x); qv[h][q8 * 8 + 1] = bf16_hi(w.x);
            qv[h][q8 * 8 + 2] = bf16_lo(w.y); qv[h][q8 * 8 + 3] = bf16_hi(w.y);
            qv[h][q8 * 8 + 4] = bf16_lo(w.z); qv[h][q8 * 8 + 5] = bf16_hi(w.z);
            qv[h][q8 * 8 + 6] = bf16_lo(w.w); qv[h][q8 * 8 + 7] = bf16_hi(w.w);
          }
        } else {
          const uint2 w = *reinterpret_cast<const uint2 *>(qs + h * kD + li * 4);
          qv[h][0] = bf16_lo(w.x); qv[h][1] = bf16_hi(w.x);
          qv[h][2] = bf16_lo(w.y); qv[h][3] = bf16_hi(w.y);
        }
      }
    }

    const uint16_t *Ks = reinterpret_cast<const uint16_t *>(stage);
    const uint16_t *Vs = Ks + kBlk * kD;
    const int rows = s_rows[bi];
    const int kw0 = warp * KW;
    const int wvalid = min(KW, rows - kw0);

    if (wvalid > 0) {
      // ---- S = q . k for this warp's keys ----
      float sv[ROUNDS];
#pragma unroll
      for (int rd = 0; rd < ROUNDS; ++rd) {
        float part[2 * R];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint16_t *krow = Ks + (kw0 + rd * KPR + kk * KG + kg) * kD;
          float kf[DS];
          if constexpr (DS >= 8) {
#pragma unroll
            for (int q8 = 0; q8 < DS / 8; ++q8) {
              const uint4 w = *reinterpret_cast<const uint4 *>(krow + (q8 * LPK + li) * 8);
              kf[q8 * 8 + 0] = bf16_lo(w.x); kf[q8 * 8 + 1] = bf16_hi(w.x);
              kf[q8 * 8 + 2] = bf16_lo(w.y); kf[q8 * 8 + 3] = bf16_hi(w.y);
              kf[q8 * 8 + 4] = bf16_lo(w.z); kf[q8 * 8 + 5] = bf16_hi(w.z);
              kf[q8 * 8 + 6] = bf16_lo(w.w); kf[q8 * 8 + 7] = bf16_hi(w.w);
            }
          } else {
            const uint2 w = *reinterpret_cast<const uint2 *>(krow + li * 4);
            kf[0] = bf16_lo(w.x); kf[1] = bf16_hi(w.x);
            kf[2] = bf16_lo(w.y); kf[3] = bf16_hi(w.y);
          }
#pragma unroll
          for (int h = 0; h < R; ++h) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < DS; ++e) s = fmaf(qv[h][e], kf[e], s);
            part[kk * R + h] = s;
          }
        }
        const float s = transpose_reduce<2 * R>(part, li);
        const int key = kw0 + rd * KPR + my_kappa * KG + kg;
        sv[rd] = key < rows ? s * a.scale_log2 : -INFINITY;
      }

      // ---- online softmax for head my_head over this warp's keys ----
      float mb = sv[0];
#pragma unroll
      for (int rd = 1; rd < ROUNDS; ++rd) mb = fmaxf(mb, sv[rd]);
      mb = warp_max_xor(mb, R, 32);  // lanes sharing a head differ in bits >= log2(R)
      const float m_new = fmaxf(m_run, mb);
      const float corr = (m_new == -INFINITY) ? 1.f : exp2f(m_run - m_new);
      float ps = 0.f;
#pragma unroll
      for (int rd = 0; rd < ROUNDS; ++rd) {
        const float pv = (sv[rd] == -INFINITY) ? 0.f : exp2f(sv[rd] - m_new);
        ps += pv;
        pw[(rd * KPR + my_kappa * KG + kg) * R + my_head] = pv;
      }
      ps = warp_sum_xor(ps, R, 32);
      l_run = l_run * corr + ps;
      m_run = m_new;
      if (lane < R) alpha[lane] = corr;  // lanes 0..R-1 hold heads 0..R-1
      __syncwarp();

      // ---- O = corr * O + P V ----
#pragma unroll
      for (int h = 0; h < R; ++h) {
        const float al = alpha[h];
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[h][e] *= al;
      }
#pragma unroll 4
      for (int kk = 0; kk < wvalid; ++kk) {
        const uint2 w = *reinterpret_cast<const uint2 *>(Vs + (kw0 + kk) * kD + lane * 4);
        const float v0 = bf16_lo(w.x), v1 = bf16_hi(w.x), v2 = bf16_lo(w.y), v3 = bf16_hi(w.y);
        const float *prow = pw + kk * R;
#pragma unroll
        for (int h = 0; h < R; ++h) {
          const float p = prow[h];
          acc[h][0] = fmaf(p, v0, acc[h][0]);
          acc[h][1] = fmaf(p, v1, acc[h][1]);
          acc[h][2] = fmaf(p, v2, acc[h][2]);
          acc[h][3] = fmaf(p, v3, acc[h][3]);
        }
      }
      __syncwarp();
    }
    __syncthreads();  // stage st fully consumed
    if (tid == 0 && bi + NSTAGE < nb) issue(bi + NSTAGE);
  }

  if (abort_at >= 0) {
    // a copy never completed: give the ones still in flight a bounded chance
    // to land before the CTA's shared memory is released, then leave
    if (tid == 0)
      for (int bj = abort_at; bj < min(nb, abort_at + NSTAGE); ++bj)
        (void)mbar_wait_bounded(&full_bar[bj % NSTAGE], (uint32_t)((bj / NSTAGE) & 1));
    __syncthreads();
    return;
  }
  for (int f = next_flush; f < n_seg; ++f) flush(f, f == cur);
}

template <int R, int NWARP, int NSTAGE>
cudaError_t launch_r(const DecArgs &a, long long grid, cudaStream_t stream) {
  const size_t smem = Cfg<R, NWARP>::smem(NSTAGE);
  auto kern = attn_streamk_kernel<R, NWARP, NSTAGE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)grid, NWARP * 32, smem, stream>>>(a);
  return cudaGetLastError();
}

int max_entries_per_cta(int R) { return R == 1 ? 2 * 64 : 2 * 128; }

}  // namespace

DecodePlan plan_gather(const sparda_params &p, long long pairs) {
  DecodePlan pl{};
  pl.S = p.k + p.n_init + p.n_local;
  const int R = p.G > 0 ? p.Hq / p.G : 1;
  const long long E = pairs * pl.S;
  long long C = kGridTarget;
  const int forced = env_int("SPARDA_DECODE_CTAS");
  if (forced > 0) C = forced;
  C = std::max<long long>(C, ceil_div_ll(E, max_entries_per_cta(R)));
  if (C > E) C = E;
  if (C < 1) C = 1;
  pl.n_cta = C;
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
  DecArgs a;
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.bg_stride = bg_stride;
  a.blk_stride = blk_stride;
  a.idx = idx;
  a.O = O;
  a.status = dev_status;
  a.n_entries = pairs * pl.S;
  a.G = p.G;
  a.S = pl.S;
  a.NB = (p.T + kBlk - 1) / kBlk;
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
    case 1: return launch_r<1, 2, 4>(a, pl.n_cta, stream);
    case 2: return launch_r<2, 4, 3>(a, pl.n_cta, stream);
    case 4: return launch_r<4, 4, 3>(a, pl.n_cta, stream);
    case 8: return launch_r<8, 4, 2>(a, pl.n_cta, stream);
    case 16: return launch_r<16, 4, 2>(a, pl.n_cta, stream);
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
