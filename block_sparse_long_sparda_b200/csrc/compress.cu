// compress.cu -- mean-pooled compressed keys (one per block of 64 tokens).
//
// Pages cited: [p4 <section>] = the article "SparDA: a fourth projection that
// lets sparse attention prefetch its own KV cache" (ai.thesatyajit.com);
// [p1 <section>] = the SparDA summary page at deepresearch2agi.pages.dev.
//
// [p1 "架构细节"]: the top-k part of a layer's block set is scored against the
// block-mean of that layer's keys; [p4 "The problem InfLLM-V2 leaves on the
// table"]: keys are mean-pooled into one compressed key per block.
//
// Design (B200): pure HBM streaming, 1/64 of the bytes written back.  One warp
// owns one (b, g, block): lanes 0-15 cover one 256-byte key row with 16-byte
// non-allocating loads, lanes 16-31 the next row, so every load instruction of
// the warp reads two whole rows (512 contiguous bytes when rows are packed).
// Eight rows per lane are in flight before any arithmetic.  fp32 accumulation,
// one shuffle to join the two half-warps, IEEE division by the row count.
#include "common.cuh"
#include "internal.h"

namespace sparda {

namespace {

__device__ __forceinline__ void acc8(float (&a)[8], uint4 v) {
  a[0] += bf16_lo(v.x);
  a[1] += bf16_hi(v.x);
  a[2] += bf16_lo(v.y);
  a[3] += bf16_hi(v.y);
  a[4] += bf16_lo(v.z);
  a[5] += bf16_hi(v.z);
  a[6] += bf16_lo(v.w);
  a[7] += bf16_hi(v.w);
}

// An item is a run of `rows` positions starting at j * step: a block (rows =
// step = 64) or a window of the window grid (rows = 32, step = 16); NB items
// per (b, g).
template <bool kContig>
__global__ void __launch_bounds__(256, 3) compress_kernel(const uint16_t *__restrict__ K,
                                                       long long bg_stride, long long tok_stride,
                                                       int T, int NB, long long n_items,
                                                       float *__restrict__ kc32,
                                                       uint16_t *__restrict__ kc16, int rows,
                                                       int step, const int32_t *seq_len, int G) {
  const int lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (item >= n_items) return;
  const long long bg = item / NB;
  const int j = (int)(item - bg * NB);
  const int t0 = j * step;
  // per-sequence lengths: a block past its sequence's end, or a window not
  // complete inside it, is left untouched
  const int Tb = seq_len ? min(T, seq_len[bg / G]) : T;
  const int n = min(rows, Tb - t0);
  if (n <= 0 || (rows != step && n < rows)) return;
  const int half = lane >> 4;
  const int c8 = lane & 15;
  if (kContig) tok_stride = kD;  // rows packed: constant offsets, fewer live registers
  const uint16_t *base = K + bg * bg_stride + (long long)t0 * tok_stride + c8 * 8;

  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (n == kBlk) {
#pragma unroll
    for (int r0 = 0; r0 < kBlk / 2; r0 += 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = ldg_stream(base + (long long)(2 * (r0 + u) + half) * tok_stride);
#pragma unroll
      for (int u = 0; u < 8; ++u) acc8(a, v[u]);
    }
  } else {
    for (int t = half; t < n; t += 2) acc8(a, ldg_stream(base + (long long)t * tok_stride));
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) a[e] += __shfl_xor_sync(0xffffffffu, a[e], 16);
  if (half) return;

  const float fn = (float)n;
  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = a[e] / fn;
  if (kc32) {
    float4 *o = reinterpret_cast<float4 *>(kc32 + item * kD + c8 * 8);
    o[0] = make_float4(m[0], m[1], m[2], m[3]);
    o[1] = make_float4(m[4], m[5], m[6], m[7]);
  }
  if (kc16) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(m[2 * e]));
      uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(m[2 * e + 1]));
      w[e] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4 *>(kc16 + item * kD + c8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// One decode token appended: write its K and V rows at position `pos` (with
// per-sequence lengths, at each sequence's last position) and
// recompute the compressed key of its block -- the one block whose mean
// changes.  One warp per (b, g).  The block's earlier rows are summed from
// memory in the same per-half, ascending-row order as compress_kernel and
// the new row is added last in its half, so the result is bit-identical to
// compressing the whole cache again.
__global__ void __launch_bounds__(256) append_kernel(const uint16_t *__restrict__ K_new,
                                                     const uint16_t *__restrict__ V_new,
                                                     uint16_t *__restrict__ K,
                                                     uint16_t *__restrict__ V, long long bg_stride,
                                                     long long blk_stride, int pos, int NB,
                                                     long long n_pairs, float *__restrict__ kc32,
                                                     uint16_t *__restrict__ kc16,
                                                     const int32_t *seq_len, int G, int T) {
  const int lane = threadIdx.x & 31;
  const long long bg = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  // launched as a programmatic dependent: everything waits for the previous
  // kernel (which may read the cache this writes)
  pdl_trigger();
  pdl_wait();
  if (bg >= n_pairs) return;
  if (seq_len) {  // per-sequence lengths: the new token is the sequence's last one
    const int len = seq_len[bg / G];
    if (len < 1 || len > T) return;  // an invalid length: nothing is appended
    pos = len - 1;
  }
  const int half = lane >> 4, c8 = lane & 15;
  const int c = pos / kBlk, r = pos - c * kBlk;  // block and row of the new token
  const long long blk_off = bg * bg_stride + (long long)c * blk_stride + c8 * 8;
  const uint4 knew = ldg_plain(K_new + bg * kD + c8 * 8);
  if (half == 0) {
    *reinterpret_cast<uint4 *>(K + blk_off + (long long)r * kD) = knew;
  } else {
    *reinterpret_cast<uint4 *>(V + blk_off + (long long)r * kD) = ldg_plain(V_new + bg * kD + c8 * 8);
  }
  // rows 0 .. r-1 of the block were written before this launch; eight rows
  // per half-warp are loaded at once and added in ascending order
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
  for (int t0 = half; t0 < r; t0 += 16) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (t0 + 2 * u < r) v[u] = ldg_plain(K + blk_off + (long long)(t0 + 2 * u) * kD);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (t0 + 2 * u < r) acc8(a, v[u]);
  }
  if ((r & 1) == half) acc8(a, knew);
#pragma unroll
  for (int e = 0; e < 8; ++e) a[e] += __shfl_xor_sync(0xffffffffu, a[e], 16);
  if (half) return;
  const float fn = (float)(r + 1);
  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = a[e] / fn;
  const long long item = bg * NB + c;
  if (kc32) {
    float4 *o = reinterpret_cast<float4 *>(kc32 + item * kD + c8 * 8);
    o[0] = make_float4(m[0], m[1], m[2], m[3]);
    o[1] = make_float4(m[4], m[5], m[6], m[7]);
  }
  if (kc16) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(m[2 * e]));
      uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(m[2 * e + 1]));
      w[e] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4 *>(kc16 + item * kD + c8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// One decode token appended, window grid: if the token at `pos` (with
// per-sequence lengths, each sequence's last position) completes a window --
// pos = w*16 + 31 -- write that window's mean.  Rows are read through the
// cache's block layout, so the interleaved K|V blocks work too.  The sum
// runs in compress_kernel's order (even rows in one half-warp, odd rows in
// the other, each ascending, then the halves added), so in the [T][d] layout
// the key is bit-identical to compressing the windows again.
__global__ void __launch_bounds__(256) append_window_kernel(
    const uint16_t *__restrict__ K, long long bg_stride, long long blk_stride, int pos, int NW,
    long long n_pairs, float *__restrict__ kw32, uint16_t *__restrict__ kw16,
    const int32_t *seq_len, int G, int T) {
  constexpr int kWin = 32, kStride = 16;
  const int lane = threadIdx.x & 31;
  const long long bg = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_trigger();
  pdl_wait();  // the new row was written by the previous kernel (sparda_append_kv)
  if (bg >= n_pairs) return;
  if (seq_len) {
    const int len = seq_len[bg / G];
    if (len < 1 || len > T) return;  // an invalid length: nothing is appended
    pos = len - 1;
  }
  if (pos < kWin - 1 || (pos - (kWin - 1)) % kStride != 0) return;  // no window ends here
  const int w = (pos - (kWin - 1)) / kStride;
  if (w >= NW) return;
  const int half = lane >> 4, c8 = lane & 15;
  const uint16_t *base = K + bg * bg_stride + c8 * 8;
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  uint4 v[kWin / 2];
#pragma unroll
  for (int u = 0; u < kWin / 2; ++u) {
    const int t = w * kStride + 2 * u + half;
    v[u] = ldg_plain(base + (long long)(t / kBlk) * blk_stride + (long long)(t % kBlk) * kD);
  }
#pragma unroll
  for (int u = 0; u < kWin / 2; ++u) acc8(a, v[u]);
#pragma unroll
  for (int e = 0; e < 8; ++e) a[e] += __shfl_xor_sync(0xffffffffu, a[e], 16);
  if (half) return;
  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = a[e] / (float)kWin;
  const long long item = bg * NW + w;
  if (kw32) {
    float4 *o = reinterpret_cast<float4 *>(kw32 + item * kD + c8 * 8);
    o[0] = make_float4(m[0], m[1], m[2], m[3]);
    o[1] = make_float4(m[4], m[5], m[6], m[7]);
  }
  if (kw16) {
    uint32_t q[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(m[2 * e]));
      uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(m[2 * e + 1]));
      q[e] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4 *>(kw16 + item * kD + c8 * 8) = make_uint4(q[0], q[1], q[2], q[3]);
  }
}

}  // namespace

cudaError_t launch_append_windows(const sparda_params &p, int pos, const uint16_t *K,
                                  long long bg_stride, long long blk_stride, float *kw32,
                                  uint16_t *kw16, cudaStream_t stream) {
  const long long pairs = (long long)p.B * p.G;
  if (pairs == 0) return cudaSuccess;
  const int warps = 8;
  const cudaError_t e =
      launch_pdl(append_window_kernel, (unsigned)ceil_div_ll(pairs, warps), warps * 32, 0, stream, K,
                 bg_stride, blk_stride, pos, window_count(p.T), pairs, kw32, kw16, p.seq_len, p.G,
                 p.T);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_compress(const sparda_params &p, const uint16_t *K, long long bg_stride,
                            long long tok_stride, float *kc32, uint16_t *kc16,
                            cudaStream_t stream) {
  return launch_compress_runs(p, K, bg_stride, tok_stride, kBlk, kBlk, kc32, kc16, stream);
}

cudaError_t launch_compress_runs(const sparda_params &p, const uint16_t *K, long long bg_stride,
                                 long long tok_stride, int rows, int step, float *kc32,
                                 uint16_t *kc16, cudaStream_t stream) {
  // blocks: ceil(T / 64) (the last may be partial); windows: complete ones
  const int NB = rows == step ? (p.T + step - 1) / step : (p.T >= rows ? (p.T - rows) / step + 1 : 0);
  const long long items = (long long)p.B * p.G * NB;
  if (items == 0) return cudaSuccess;
  const int warps = 8;
  const long long grid = ceil_div_ll(items, warps);
  if (tok_stride == kD)
    compress_kernel<true><<<(unsigned)grid, warps * 32, 0, stream>>>(
        K, bg_stride, tok_stride, p.T, NB, items, kc32, kc16, rows, step, p.seq_len, p.G);
  else
    compress_kernel<false><<<(unsigned)grid, warps * 32, 0, stream>>>(
        K, bg_stride, tok_stride, p.T, NB, items, kc32, kc16, rows, step, p.seq_len, p.G);
  return cudaGetLastError();
}

cudaError_t launch_append(const sparda_params &p, int pos, const uint16_t *K_new,
                          const uint16_t *V_new, uint16_t *K, uint16_t *V, long long bg_stride,
                          long long blk_stride, float *kc32, uint16_t *kc16, cudaStream_t stream) {
  const long long pairs = (long long)p.B * p.G;
  if (pairs == 0) return cudaSuccess;
  const int NB = (p.T + kBlk - 1) / kBlk;
  const int warps = 8;
  const cudaError_t e =
      launch_pdl(append_kernel, (unsigned)ceil_div_ll(pairs, warps), warps * 32, 0, stream, K_new,
                 V_new, K, V, bg_stride, blk_stride, pos, NB, pairs, kc32, kc16, p.seq_len, p.G, p.T);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sparda
