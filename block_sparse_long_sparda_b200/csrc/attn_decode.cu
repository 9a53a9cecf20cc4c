// attn_decode.cu -- GQA block-sparse decode attention.
//
// [p4 "The fourth projection", Eq. 5 / Algorithm 2]: O_l = attention(Q_l,
// K_l[B_l], V_l[B_l]): the decode query of each head attends over the keys
// of its GQA group's selected blocks only; fp32 softmax and accumulation.
//
// Design (B200).  Decode attention reads 32 KB of K+V per selected block and
// does 2*R*128 fp32 FMA per key (R query heads share each key), about 4
// FLOP/byte for R = 4: firmly HBM bound, so CUDA cores do the math and the
// work is organised around keeping HBM busy:
//  - split-KV: a thread block owns `bps` consecutive entries of one (b, g)
//    list; thousands of thread blocks stream blocks concurrently;
//  - each selected block is staged by the bulk-copy engine
//    (cp.async.bulk global->shared, completion on an mbarrier) into an
//    NSTAGE-deep ring, so up to NSTAGE*32 KB per CTA are in flight with no
//    register cost;
//  - the 64 keys of a staged block are split over the warps; within a warp,
//    QK^T keeps each lane's slice of the R query vectors in registers (64
//    floats), every lane converts only its own K elements, and a butterfly
//    transpose-reduce turns per-lane partials into whole dot products with
//    one shuffle per (key, head) pair;
//  - online softmax (exp2 domain) per warp, P through a 1 KB shared tile,
//    PV with each lane owning 4 output dims of all R heads;
//  - warps merge in shared memory; splits merge in a small combine kernel.
// Waits on the mbarriers are bounded; a timeout sets SPARDA_DEV_TIMEOUT and
// the block leaves uniformly.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sparda {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kStageBytes = 2 * kBlk * kD * 2;  // K + V of one block = 32 KB
constexpr int kMaxBps = 128;

struct DecArgs {
  const uint16_t *Q, *K, *V;
  long long bg_stride, blk_stride;
  const int32_t *idx;
  uint16_t *O;
  float *ws_o;   // [pairs][n_split][R][128]
  float2 *ws_ml; // [pairs][n_split][R]
  int32_t *status;
  int G, S, bps, n_split, NB, addr_mode;
  int nq, q_start;  // query token i of a sequence sits at q_start + i
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

template <int R, int NWARP, int NSTAGE>
__global__ void __launch_bounds__(NWARP * 32) attn_decode_kernel(DecArgs a) {
  constexpr int DS = 64 / R;          // q dims per lane in QK
  constexpr int LPK = 2 * R;          // lanes per key in QK
  constexpr int KG = 32 / LPK;        // key groups per warp
  constexpr int KW = kBlk / NWARP;    // keys per warp per block
  constexpr int KPR = 2 * KG;         // keys per warp per QK round
  constexpr int ROUNDS = KW / KPR;
  static_assert(ROUNDS >= 1 && KW % KPR == 0, "bad warp split");
  static_assert(DS >= 4, "R too large");

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *stages = smem;                                               // NSTAGE x 32 KB
  float *pbuf = reinterpret_cast<float *>(smem + NSTAGE * kStageBytes); // NWARP x (KW*R + R)
  __shared__ __align__(8) uint64_t full_bar[NSTAGE];
  __shared__ int s_m[kMaxBps];
  __shared__ int s_rows[kMaxBps];
  __shared__ int s_nb;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // a "pair" is one (sequence, query token, group): index (b*nq + i)*G + g
  const long long pair = blockIdx.x / a.n_split;
  const int split = (int)(blockIdx.x - pair * a.n_split);
  const int g = (int)(pair % a.G);
  const long long bi = pair / a.G;
  const long long b = bi / a.nq;
  const int pos = a.q_start + (int)(bi % a.nq);
  const int c = pos / kBlk;

  // ---- this split's valid blocks ----
  if (tid == 0) {
    int nb = 0;
    const int s0 = split * a.bps, s1 = min(a.S, s0 + a.bps);
    for (int s = s0; s < s1; ++s) {
      const int j = a.idx[(long long)pair * a.S + s];
      if (j < 0) continue;
      if (j >= a.NB || j > c) {
        flag_status(a.status, SPARDA_DEV_RANGE);
        continue;
      }
      s_m[nb] = a.addr_mode == SPARDA_ADDR_SLOT ? s : j;
      s_rows[nb] = min(kBlk, pos + 1 - j * kBlk);
      ++nb;
    }
    s_nb = nb;
    for (int st = 0; st < NSTAGE; ++st) mbar_init(&full_bar[st], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int nb = s_nb;
  const uint16_t *Kbg = a.K + (b * a.G + g) * a.bg_stride;
  const uint16_t *Vbg = a.V + (b * a.G + g) * a.bg_stride;

  auto issue = [&](int bi) {
    const int st = bi % NSTAGE;
    const uint32_t bytes = (uint32_t)s_rows[bi] * kD * 2;
    uint8_t *dst = stages + st * kStageBytes;
    const long long off = (long long)s_m[bi] * a.blk_stride;
    mbar_arrive_expect_tx(&full_bar[st], 2 * bytes);
    bulk_g2s(dst, Kbg + off, bytes, &full_bar[st]);
    bulk_g2s(dst + kStageBytes / 2, Vbg + off, bytes, &full_bar[st]);
  };
  if (tid == 0)
    for (int bi = 0; bi < min(nb, NSTAGE); ++bi) issue(bi);

  // ---- per-lane query slice: qv[h][e] = q_h[dim(e)] ----
  const int kg = lane / LPK, li = lane % LPK;
  const uint16_t *qbase = a.Q + pair * R * kD;  // [..][Hq][d] with Hq = G*R
  float qv[R][DS];
#pragma unroll
  for (int h = 0; h < R; ++h) {
    if constexpr (DS >= 8) {
#pragma unroll
      for (int q8 = 0; q8 < DS / 8; ++q8) {
        const uint4 w = *reinterpret_cast<const uint4 *>(qbase + h * kD + (q8 * LPK + li) * 8);
        qv[h][q8 * 8 + 0] = bf16_lo(w.x); qv[h][q8 * 8 + 1] = bf16_hi(w.x);
        qv[h][q8 * 8 + 2] = bf16_lo(w.y); qv[h][q8 * 8 + 3] = bf16_hi(w.y);
        qv[h][q8 * 8 + 4] = bf16_lo(w.z); qv[h][q8 * 8 + 5] = bf16_hi(w.z);
        qv[h][q8 * 8 + 6] = bf16_lo(w.w); qv[h][q8 * 8 + 7] = bf16_hi(w.w);
      }
    } else {
      const uint2 w = *reinterpret_cast<const uint2 *>(qbase + h * kD + li * 4);
      qv[h][0] = bf16_lo(w.x); qv[h][1] = bf16_hi(w.x);
      qv[h][2] = bf16_lo(w.y); qv[h][3] = bf16_hi(w.y);
    }
  }

  float m_run = -INFINITY, l_run = 0.f;  // for head (li % R)
  float acc[R][4];
#pragma unroll
  for (int h = 0; h < R; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;

  float *pw = pbuf + warp * (KW * R + R);
  float *alpha = pw + KW * R;
  const int my_head = li % R;
  const int my_kappa = li / R;

  int abort_at = -1;
#pragma unroll 1
  for (int bi = 0; bi < nb; ++bi) {
    const int st = bi % NSTAGE;
    const bool ok = mbar_wait_bounded(&full_bar[st], (uint32_t)((bi / NSTAGE) & 1));
    if (!ok) flag_status(a.status, SPARDA_DEV_TIMEOUT);
    if (__syncthreads_or(!ok)) {
      abort_at = bi;
      break;
    }

    const uint16_t *Ks = reinterpret_cast<const uint16_t *>(stages + st * kStageBytes);
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
          const int key = kw0 + rd * KPR + kk * KG + kg;
          const uint16_t *krow = Ks + key * kD;
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
        const int key = rd * KPR + my_kappa * KG + kg;  // key within the warp
        pw[key * R + my_head] = pv;
      }
      ps = warp_sum_xor(ps, R, 32);
      l_run = l_run * corr + ps;
      m_run = m_new;
      if (lane < R) alpha[lane] = corr;  // lanes 0..R-1 hold heads 0..R-1
      __syncwarp();

      // ---- O = corr * O + P V ----
      float al[R];
#pragma unroll
      for (int h = 0; h < R; ++h) al[h] = alpha[h];
#pragma unroll
      for (int h = 0; h < R; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[h][e] *= al[h];
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
    // to land before the block's shared memory is released, then leave
    if (tid == 0)
      for (int bj = abort_at; bj < min(nb, abort_at + NSTAGE); ++bj)
        (void)mbar_wait_bounded(&full_bar[bj % NSTAGE], (uint32_t)((bj / NSTAGE) & 1));
    __syncthreads();
    return;
  }
  __syncthreads();

  // ---- merge the warps (stage memory is free now) ----
  float *red_o = reinterpret_cast<float *>(stages);          // [NWARP][R][128]
  float *red_m = red_o + NWARP * R * kD;                     // [NWARP][R]
  float *red_l = red_m + NWARP * R;                          // [NWARP][R]
#pragma unroll
  for (int h = 0; h < R; ++h)
    *reinterpret_cast<float4 *>(red_o + (warp * R + h) * kD + lane * 4) =
        make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
  if (lane < R) {
    red_m[warp * R + lane] = m_run;
    red_l[warp * R + lane] = l_run;
  }
  __syncthreads();

  for (int t = tid; t < R * kD; t += NWARP * 32) {
    const int h = t / kD, dim = t % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) M = fmaxf(M, red_m[w * R + h]);
    float L = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) {
      const float mw = red_m[w * R + h];
      const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
      L += f * red_l[w * R + h];
      o += f * red_o[(w * R + h) * kD + dim];
    }
    if (a.n_split == 1) {
      const float r = L > 0.f ? o / L : 0.f;
      a.O[(pair * R + h) * kD + dim] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
    } else {
      const long long ps = pair * a.n_split + split;
      a.ws_o[(ps * R + h) * kD + dim] = o;
      if (dim == 0) a.ws_ml[ps * R + h] = make_float2(M, L);
    }
  }
}

template <int R>
__global__ void __launch_bounds__(128) attn_decode_combine(const float *__restrict__ ws_o,
                                                           const float2 *__restrict__ ws_ml,
                                                           int n_split, uint16_t *__restrict__ O) {
  const long long pair = blockIdx.x;
  const int dim = threadIdx.x;
#pragma unroll 1
  for (int h = 0; h < R; ++h) {
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, ws_ml[(pair * n_split + s) * R + h].x);
    float L = 0.f, o = 0.f;
    for (int s = 0; s < n_split; ++s) {
      const long long ps = pair * n_split + s;
      const float2 ml = ws_ml[ps * R + h];
      const float f = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
      L += f * ml.y;
      o += f * ws_o[(ps * R + h) * kD + dim];
    }
    const float r = L > 0.f ? o / L : 0.f;
    O[(pair * R + h) * kD + dim] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
  }
}

template <int R, int NWARP, int NSTAGE>
cudaError_t launch_r(const DecArgs &a, long long pairs, cudaStream_t stream) {
  constexpr int KW = kBlk / NWARP;
  const size_t smem = (size_t)NSTAGE * kStageBytes + (size_t)NWARP * (KW * R + R) * 4;
  auto kern = attn_decode_kernel<R, NWARP, NSTAGE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)(pairs * a.n_split), NWARP * 32, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.n_split == 1) return e;
  attn_decode_combine<R><<<(unsigned)pairs, 128, 0, stream>>>(a.ws_o, a.ws_ml, a.n_split, a.O);
  return cudaGetLastError();
}

constexpr int kStages = 3;

}  // namespace

DecodePlan plan_gather(const sparda_params &p, long long pairs) {
  DecodePlan pl{};
  pl.S = p.k + p.n_init + p.n_local;
  int bps = env_int("SPARDA_DECODE_BPS");
  if (bps <= 0) {
    // enough thread blocks for ~4 waves of 2 resident CTAs per SM
    const long long want = 8LL * 148;
    long long n_split = pairs > 0 ? ceil_div_ll(want, pairs) : 1;
    if (n_split < 1) n_split = 1;
    bps = (int)ceil_div_ll(pl.S, n_split);
    if (bps < 2) bps = 2;
  }
  if (bps > kMaxBps) bps = kMaxBps;
  pl.bps = bps;
  pl.n_split = (int)ceil_div_ll(pl.S, bps);
  const int R = p.G > 0 ? p.Hq / p.G : 1;
  pl.ws_bytes = 0;
  if (pl.n_split > 1) {
    const size_t parts = (size_t)pairs * pl.n_split * R;
    pl.ws_bytes = ((parts * kD * 4 + 255) & ~(size_t)255) + parts * 8;
  }
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
  a.G = p.G;
  a.S = pl.S;
  a.bps = pl.bps;
  a.n_split = pl.n_split;
  a.NB = (p.T + kBlk - 1) / kBlk;
  a.addr_mode = addr_mode;
  a.nq = nq;
  a.q_start = q_start;
  const float scale = p.scale > 0.f ? p.scale : 1.0f / sqrtf((float)p.d);
  a.scale_log2 = scale * kLog2e;
  a.ws_o = nullptr;
  a.ws_ml = nullptr;
  if (pl.n_split > 1) {
    const size_t parts = (size_t)pairs * pl.n_split * R;
    a.ws_o = static_cast<float *>(ws);
    a.ws_ml = reinterpret_cast<float2 *>(static_cast<char *>(ws) +
                                         ((parts * kD * 4 + 255) & ~(size_t)255));
  }
  switch (R) {
    case 1: return launch_r<1, 2, kStages>(a, pairs, stream);
    case 2: return launch_r<2, 4, kStages>(a, pairs, stream);
    case 4: return launch_r<4, 4, kStages>(a, pairs, stream);
    case 8: return launch_r<8, 4, kStages>(a, pairs, stream);
    case 16: return launch_r<16, 4, kStages>(a, pairs, stream);
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
