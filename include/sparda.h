/*
 * sparda.h -- C ABI of libsparda, the B200 (sm_100a) hot path of SparDA
 * (Sparse Decoupled Attention): Forecast-driven lookahead block selection
 * plus GQA block-sparse attention.
 *
 * Sources: "SparDA: a fourth projection that lets sparse attention prefetch
 * its own KV cache" (ai.thesatyajit.com/articles/sparda) -- cited below as
 * [p4 <section>] -- and deepresearch2agi.pages.dev/sparda_sparse_decoupled_attention
 * -- cited as [p1 <section>].
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Return value: SPARDA_OK (0) or a negative status below.  Arguments are
 *    validated on the host before anything is enqueued; a call that returns
 *    an error has enqueued nothing, except SPARDA_ECUDA, which reports a
 *    launch failure (cudaGetLastError after the launch; the call never
 *    synchronizes).
 *  - Calls are asynchronous on the given stream (a cudaStream_t; NULL means
 *    the legacy default stream).  Results depend only on the arguments: the
 *    library reads no environment variables and keeps no state between calls
 *    beyond per-device kernel attributes it caches on first use (and the
 *    fixed scratch array of the allocation-free entry point below).  Calls
 *    on different streams with disjoint buffers may run concurrently.
 *  - All buffers are owned by the caller.  Device buffers are plain device
 *    pointers; every pointer must be 16-byte aligned and every row stride a
 *    multiple of 8 elements (16 bytes).
 *  - bf16 tensors are passed as `const void *` to raw IEEE bfloat16 storage.
 *  - Layouts are row-major, innermost index last.  Query head h belongs to
 *    KV group (GQA group) h / (Hq / G).
 *  - Supported shapes in this version: d = 128, blk = 64, Hq / G in
 *    {1, 2, 4, 8, 16}; other values return SPARDA_EUNSUPPORTED.
 *  - Block j of a sequence holds token positions [j*blk, (j+1)*blk).
 *    NB = ceil(T / blk).  For a query at position pos, c = pos / blk is its
 *    own block; its set is B = init U local U topk [p4 "The problem
 *    InfLLM-V2 leaves on the table", eq. B_l(i)] with
 *      local = [max(0, c - n_local + 1), c],
 *      init  = [0, n_init) minus the local blocks,
 *      topk  = the k best-scoring candidate blocks [n_init, c - n_local + 1),
 *    stored as S = k + n_init + n_local int32 block ids in ascending order,
 *    padded with -1 at the end when fewer blocks exist.
 *  - dev_status (optional, device int32): kernels OR device-side findings
 *    into it (SPARDA_DEV_RANGE: a block id outside [0, NB) or after the
 *    query's own block was skipped; SPARDA_DEV_TIMEOUT: a bounded wait gave
 *    up; SPARDA_DEV_LAYOUT: a kernel found its shared memory placed off the
 *    1024-byte boundary its swizzled tiles need and wrote nothing).  The
 *    caller zeroes it, reads it after synchronizing, and may turn
 *    it into a status with sparda_status_from_device().
 */
#ifndef SPARDA_H_
#define SPARDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *sparda_stream_t; /* == cudaStream_t */

enum sparda_status {
  SPARDA_OK = 0,
  SPARDA_EINVAL = -1,       /* null / misaligned pointer, bad shape or size          */
  SPARDA_EUNSUPPORTED = -2, /* valid but outside this version's shapes (d, blk, r)   */
  SPARDA_ECUDA = -3,        /* a CUDA call or kernel launch failed                   */
  SPARDA_ERANGE = -4,       /* device-side bounds finding (from the status word)     */
  SPARDA_ETIMEOUT = -5,     /* a bounded device-side wait gave up                    */
  SPARDA_EWORKSPACE = -6    /* workspace missing or smaller than sparda_workspace_size */
};

enum sparda_device_status_bits {
  SPARDA_DEV_RANGE = 1,
  SPARDA_DEV_TIMEOUT = 2,
  SPARDA_DEV_LAYOUT = 4
};

/* Optional launch choices the library otherwise makes itself, for tuning
 * sweeps and for tests that force each kernel variant.  A NULL
 * sparda_params.tune, or a field left 0, keeps the library's own choice; no
 * field changes what a call computes, only how.  Workspace sizes follow the
 * same params: size a workspace with the tune pointer the calls will use. */
typedef struct sparda_tuning {
  int select_chunk;   /* candidate blocks per selection thread block (rounded down
                         to a multiple of 256, at least 256)                      */
  int select_stream;  /* nonzero: query chunks of >= 64 tokens take the streaming
                         selection instead of the tensor-core score tiles         */
  int select_binned;  /* nonzero: the binned threshold search even where the
                         sorting-network threshold applies (k <= 64, <= 2048
                         candidates), and, for query chunks ranked row by row,
                         even where the listed sample threshold applies
                         (k <= 64, 1024 to 2048 candidates)                      */
  int attn_ctas;      /* attention thread blocks (kept within what the lists need
                         and the workspace was sized for)                        */
  int attn_stages;    /* attention ring depth: 2, 3, 4 or 6 stages of 32 KB       */
  int attn_split_kv;  /* 1: a ring slot's K and V tiles are refilled separately,
                         -1: together; 0: separately for prefill only            */
  int prefetch_ctas;  /* gather thread blocks when a call passes n_ctas = 0      */
  int attn_prefill_per_token;  /* nonzero: prefill attention streams each token's
                         own block list (the decode kernel, one (token, group)
                         pair per list) instead of the block-major kernels     */
  long long attn_wait_cycles;  /* bound of every wait in the attention kernel, in
                         SM clock cycles; 0: 2e9 (about one second).  Waits that
                         run out end the call with SPARDA_DEV_TIMEOUT            */
} sparda_tuning;

/* Shapes shared by every call.  T is the number of tokens present in the
 * sequence (the context length); the decode query sits at position T - 1. */
typedef struct sparda_params {
  int B;        /* batch (sequences); B = 0 is a valid empty call              */
  int Hq;       /* query heads                                                 */
  int G;        /* GQA groups = KV heads; Hq % G == 0                          */
  int d;        /* head dimension (128)                                        */
  int blk;      /* tokens per block (64)                                       */
  int T;        /* tokens present, >= 1                                        */
  int k;        /* top-k budget (>= 0, <= 1024)                                */
  int n_init;   /* initial blocks (>= 0, <= 64)                                */
  int n_local;  /* local-window blocks (>= 0, <= 64)                           */
  float scale;  /* attention logit scale; <= 0 means 1/sqrt(d)                 */
  /* Optional device int32 [B]: tokens present in each sequence, seq_len[b]
   * <= T (T then only sizes the arrays).  Null: every sequence holds T tokens.
   * With lengths, the nq query tokens of sequence b are its last nq tokens,
   * positions seq_len[b] - nq .. seq_len[b] - 1 (a decode query is the last
   * token), and the calls' q_start is not used.  Honoured by
   * sparda_compress_keys and sparda_compress_windows (blocks past the end,
   * and windows not complete inside the sequence, are left untouched),
   * sparda_forecast_select and sparda_forecast_select_windows,
   * sparda_prefetch_blocks, and the decode and prefill attention calls; the
   * cache plan and the cached prefetch follow the lists they are given;
   * sparda_append_kv and sparda_append_windows take each sequence's new
   * token at seq_len[b] - 1 (an invalid length appends nothing there).  A length
   * outside [nq, T] (nq = 1 for decode and compression) gives that sequence
   * empty outputs (-1 sets, zero attention output) and is flagged
   * SPARDA_DEV_RANGE where a status word is given. */
  const int32_t *seq_len;
  /* Optional host pointer: launch choices (see sparda_tuning); NULL: the
   * library's own.  Read during the call only. */
  const sparda_tuning *tune;
} sparda_params;

/* ops for sparda_workspace_size */
enum sparda_op {
  SPARDA_OP_COMPRESS = 0,
  SPARDA_OP_SELECT = 1,
  SPARDA_OP_PREFETCH = 2,
  SPARDA_OP_ATTN_DECODE = 3,
  SPARDA_OP_ATTN_PREFILL = 4,
  SPARDA_OP_SELECT_WINDOWS = 5,
  SPARDA_OP_HEAD_SOFTMAX = 6,         /* sparda_head_softmax_select (nq = 1)         */
  SPARDA_OP_HEAD_SOFTMAX_WINDOWS = 7  /* sparda_head_softmax_select_windows (nq = 1) */
};

/* how sparda_sparse_attn_decode finds the storage of list entry s */
enum sparda_addr_mode {
  SPARDA_ADDR_LOGICAL = 0, /* block id idx[s] indexes the K/V buffer (KV resident)   */
  SPARDA_ADDR_SLOT = 1,    /* list position s indexes it (prefetched device slots)  */
  SPARDA_ADDR_PHYS = 2     /* phys[s] indexes it (slot cache; see the cached calls) */
};

/*
 * sparda_compress_keys -- mean-pooled compressed keys.
 *   [p1 "架构细节"]: top-k blocks are scored against the block-mean of the
 *   layer's keys; [p4 "The problem InfLLM-V2 leaves on the table"]: keys are
 *   mean-pooled into one compressed key per block.
 *   Kc[b,g,j,:] = (1/n_j) sum_{t in block j, t < T} K[b,g,t,:]
 * K        bf16, row (b,g,t) at K + (b*G+g)*bg_stride + t*tok_stride (elements)
 * kc_f32   float [B][G][NB][d] or NULL
 * kc_bf16  bf16  [B][G][NB][d] or NULL (round-to-nearest-even of the fp32 mean)
 * At least one output must be non-NULL.  Accumulation is fp32.
 */
int sparda_compress_keys(const sparda_params *p, const void *K, long long bg_stride,
                         long long tok_stride, float *kc_f32, void *kc_bf16,
                         sparda_stream_t stream);

/*
 * sparda_append_kv -- one decode token: write its K and V rows at position
 * pos of every (b,g) and recompute the compressed key of the block holding
 * pos (the only block whose mean changes), so selection can run on an up to
 * date Kc without compressing the whole cache again.
 *   [p4 "The fourth projection", Algorithm 2]: kv_cache.append(K_l, V_l);
 *   k_compressed_cache.update_incremental(kv_cache).
 * K_new, V_new  bf16 [B][G][d] device, the new token's key and value rows
 * K, V     bf16 device caches; row t of (b,g) sits at
 *            base + (b*G+g)*bg_stride + (t/blk)*blk_stride + (t%blk)*d
 *          ([B][G][T][d]: bg_stride = T*d, blk_stride = blk*d; interleaved
 *          [..][NB][2][blk][d]: V = K + blk*d, blk_stride = 2*blk*d)
 * pos      the new token's position, 0 <= pos < T (T sizes the Kc arrays);
 *          not used with per-sequence lengths (p->seq_len), where sequence
 *          b's token goes to seq_len[b] - 1
 * kc_f32, kc_bf16  as for sparda_compress_keys, [B][G][NB][d]; only block
 *          pos/blk is written.  The value is bit-identical to what
 *          sparda_compress_keys computes over positions 0..pos.
 */
int sparda_append_kv(const sparda_params *p, int pos, const void *K_new, const void *V_new,
                     void *K, void *V, long long bg_stride, long long blk_stride, float *kc_f32,
                     void *kc_bf16, sparda_stream_t stream);

/*
 * sparda_forecast_select -- block sets from Forecast scores.
 *   [p4 "The fourth projection", Eq. 4]:
 *     B_{l+1} = B_init U B_local U f_top(F_l Kc_{l+1}^T, k)
 *   [p4 "One Forecast head per GQA group"]: one Forecast vector per GQA group,
 *   raw dot-product scores, top-k with no softmax.  With nf > 1 the nf
 *   vectors of a group are the group's query heads and their scores are
 *   summed: the multi-head baseline selector of the same section (whose
 *   softmax after the sum cannot change the ranking and is not applied).
 * F     bf16 [B][nq][G][nf][d]   (nf = 1: Forecast; nf = Hq/G: baseline)
 * kc    bf16 [B][G][NB][d]       compressed keys of the layer being selected
 * idx   int32 [B][nq][G][S]      output, ascending block ids, -1 padded
 * Query token i sits at position q_start + i; 0 <= q_start, q_start + nq <= T
 * (with per-sequence lengths, at seq_len[b] - nq + i: q_start is checked but
 * not used).
 * nq = 1 is the decode path; nq > 1 scores every query token (prefill).
 * Ranking: higher fp32 score first, equal scores -> lower block index.
 * ws    device workspace of sparda_workspace_size(SPARDA_OP_SELECT, p, nq, nf)
 *       bytes; it must be zero-filled before its first use, and each call
 *       leaves its tickets and flags at zero again, a call that timed out
 *       included (the rest is scratch).  Calls sharing one workspace must not
 *       overlap on the device.
 * dev_status  optional device word: SPARDA_DEV_TIMEOUT if a copy of the keys
 *       never landed within the bounded wait; the sets of the problems it hit
 *       are then written as -1 throughout (never a wrong set), and the others
 *       stay valid.  SPARDA_DEV_RANGE for an invalid per-sequence length.
 */
int sparda_forecast_select(const sparda_params *p, const void *F, int nq, int nf, int q_start,
                           const void *kc, int32_t *idx, void *ws, size_t ws_bytes,
                           int32_t *dev_status, sparda_stream_t stream);

/*
 * The window grid of the models the pages measure (f3): [p4 "One Forecast
 * head per GQA group"] -- both test models pool their keys with a 32-token
 * window at stride 16, and [p4 "Training: distilling the selector you
 * already have"] names the selector's final max-pooling of the scores to
 * blocks.  The pages do not print the window-to-block map; the one taken
 * here: block j's score is the largest score of the windows lying inside
 * it, windows 4j, 4j+1 and 4j+2 (window 4j+3 straddles two blocks).
 *
 * sparda_compress_windows -- kw[b,g,w] = mean of the keys at positions
 *   [w*stride, w*stride + win), complete windows only: NW = (T - win) /
 *   stride + 1 for T >= win.  win = 32, stride = 16 (others:
 *   SPARDA_EUNSUPPORTED); K as for sparda_compress_keys; kw_f32 / kw_bf16
 *   [B][G][NW][d] (either may be null, not both).
 */
int sparda_compress_windows(const sparda_params *p, const void *K, long long bg_stride,
                            long long tok_stride, int win, int stride, float *kw_f32,
                            void *kw_bf16, sparda_stream_t stream);

/*
 * sparda_append_windows -- the window grid's part of a decode append: once
 *   the new token's K row is in the cache (sparda_append_kv), write the key
 *   of the window that token completes, if any (pos = w*stride + win - 1).
 *   Windows that are not complete do not exist (as in
 *   sparda_compress_windows), so no other window changes.
 *   [p4 "The fourth projection", Algorithm 2] (update_incremental) on the
 *   grid of [p4 "One Forecast head per GQA group"].
 * pos, K, bg_stride, blk_stride  as for sparda_append_kv (with per-sequence
 *          lengths, sequence b's token is at seq_len[b] - 1)
 * win, stride  32 and 16 (others: SPARDA_EUNSUPPORTED)
 * kw_f32, kw_bf16  [B][G][NW][d] as for sparda_compress_windows; with the
 *          [B][G][T][d] layout the key is bit-identical to what that call
 *          computes.
 * Returns SPARDA_EINVAL for a bad pos (without lengths), pointer or stride.
 */
int sparda_append_windows(const sparda_params *p, int pos, const void *K, long long bg_stride,
                          long long blk_stride, int win, int stride, float *kw_f32, void *kw_bf16,
                          sparda_stream_t stream);

/*
 * sparda_forecast_select_windows -- sparda_forecast_select on the window
 *   grid: kw bf16 [B][G][NW][d] from sparda_compress_windows (T sets NW);
 *   a candidate block scores as the best window inside it, then the same
 *   top-k rule, tie rule and output.  ws: sparda_workspace_size(
 *   SPARDA_OP_SELECT_WINDOWS, p, nq, nf) bytes, zero-filled before first use;
 *   ws and dev_status as for sparda_forecast_select.
 */
int sparda_forecast_select_windows(const sparda_params *p, const void *F, int nq, int nf,
                                   int q_start, const void *kw, int win, int stride,
                                   int32_t *idx, void *ws, size_t ws_bytes,
                                   int32_t *dev_status, sparda_stream_t stream);

/*
 * sparda_head_softmax_select -- the original selector in its per-head softmax
 *   form, the comparator the Forecast indexer replaces.
 *   [p4 "Training: distilling the selector you already have"], Eq. 6: the
 *   original selector's shared importance score is, summed over the group's
 *   query heads, each head's softmax over the compressed keys of
 *   Q_h Kc^T / tau; the selected set is its top-k minus the initial and
 *   local blocks.  [p4 "One Forecast head per GQA group"]: the baseline
 *   scores with every query head of the group (G score products and a
 *   softmax per layer).
 *     w_r = sum_h exp(s_hr - M_h) / Z_h,  s_hr = Q_h . Kc_r / tau,
 *     M_h = max_r s_hr,  Z_h = sum_r exp(s_hr - M_h),
 *   r over every key row the query sees: blocks 0..c (c = the query's own
 *   block), or on the window grid the windows complete by the query position.
 *   The initial and local rows and the windows straddling two blocks count
 *   in Z_h but are never ranked.  Set = init U top-k(w) U local, ascending,
 *   -1 padded; equal weights go to the lower block index.  Weights are fp32
 *   (scores, exp, sums).
 * Q     bf16 [B][G][nf][d]  the decode query's heads by group, 1 <= nf <= 16
 * kc    bf16 [B][G][NB][d]  block keys
 * tau   softmax temperature; <= 0 means sqrt(d)
 * idx   int32 [B][G][S], S = k + n_init + n_local
 * One query token per sequence: at q_start (0 <= q_start < T), or with
 * per-sequence lengths the sequence's last token (q_start is checked only).
 * ws    device workspace of sparda_workspace_size(SPARDA_OP_HEAD_SOFTMAX, p,
 *       1, nf) bytes, zero-filled before its first use; each call leaves its
 *       tickets and flags at zero again, a call that timed out included (the
 *       rest is scratch).  Calls sharing one workspace must not overlap on the
 *       device.
 * dev_status  optional device word: SPARDA_DEV_TIMEOUT when a copy or a
 *       product never completed within the bounded wait (that problem's set
 *       is written as -1 throughout), SPARDA_DEV_RANGE for an invalid
 *       per-sequence length (also an empty set), SPARDA_DEV_LAYOUT if shared
 *       memory was misplaced.
 */
int sparda_head_softmax_select(const sparda_params *p, const void *Q, int nf, int q_start,
                               float tau, const void *kc, int32_t *idx, void *ws,
                               size_t ws_bytes, int32_t *dev_status, sparda_stream_t stream);

/*
 * sparda_head_softmax_select_windows -- the same on the window grid: kw bf16
 *   [B][G][NW][d] window keys (win = 32, stride = 16, NW as
 *   sparda_compress_windows gives for T), and a block weighs as much as the
 *   heaviest of the windows inside it (windows 4j, 4j+1, 4j+2; -inf for a
 *   block with none), the selector's final max-pooling
 *   [p4 "Training: distilling the selector you already have"].  Workspace op
 *   SPARDA_OP_HEAD_SOFTMAX_WINDOWS; ws and dev_status as for
 *   sparda_head_softmax_select.
 */
int sparda_head_softmax_select_windows(const sparda_params *p, const void *Q, int nf,
                                       int q_start, float tau, const void *kw, int win,
                                       int stride, int32_t *idx, void *ws, size_t ws_bytes,
                                       int32_t *dev_status, sparda_stream_t stream);

/*
 * sparda_prefetch_blocks -- gather the selected K/V blocks of one layer from
 * page-locked host memory into device slots, read by the GPU over the
 * host link (zero-copy), so the block ids never travel back to the host.
 *   [p4 "The fourth projection", Algorithm 2]: fetch(B_next, src = CPU
 *   pinned, dst = GPU) launched on a dedicated prefetch stream; [p1
 *   "UVA异步预取管线"]: the number of thread blocks adapts to the batch.
 * host_kv  bf16 [B][G][NB][2][blk][d] (K block then V block), page-locked
 *          and mapped (cudaHostAlloc(..., cudaHostAllocMapped) or
 *          cudaHostRegister(..., cudaHostRegisterMapped)); the host pointer
 *          is translated with cudaPointerGetAttributes.  Not pinned/mapped
 *          -> SPARDA_EINVAL.
 * idx      int32 [B][G][S] device, the layer's block sets (decode position T-1)
 * slots    bf16 [B][G][S][2][blk][d] device; slot s receives block idx[s]
 * skip_resident  nonzero: initial and local entries are not copied (the
 *          caller keeps them resident in their slots); -1 entries never are.
 * n_ctas   thread blocks to use, 0 = chosen from B
 * A block id outside [0, NB) is skipped and flagged SPARDA_DEV_RANGE.
 */
int sparda_prefetch_blocks(const sparda_params *p, const void *host_kv, const int32_t *idx,
                           void *slots, int skip_resident, int n_ctas, int32_t *dev_status,
                           sparda_stream_t stream);

/*
 * sparda_sparse_attn_decode -- one decode query per sequence attends over
 * the keys of its group's block set only, fp32 softmax and accumulation.
 *   [p4 "The fourth projection", Eq. 5 / Algorithm 2]:
 *     O_l = attention(Q_l, K_l[B_l], V_l[B_l])
 * Q     bf16 [B][Hq][d], query at position T-1
 * K, V  bf16; the block stored for list entry s of (b,g) starts at
 *         base + (b*G+g)*bg_stride + m*blk_stride   (elements)
 *       with m = idx[b,g,s] (SPARDA_ADDR_LOGICAL) or m = s (SPARDA_ADDR_SLOT);
 *       its blk rows are contiguous (row stride d).  Separate [B][G][T][d]
 *       tensors: bg_stride = T*d, blk_stride = blk*d.  Interleaved
 *       [..][2][blk][d] storage: V = K + blk*d, blk_stride = 2*blk*d.
 * idx   int32 [B][G][S]; keys after position T-1 are masked; -1 skipped.
 *       A list must not repeat a block.
 * O     bf16 [B][Hq][d]
 * ws    device workspace of sparda_workspace_size(SPARDA_OP_ATTN_DECODE, ...)
 *       bytes, zero-filled before its first use (each call leaves its ticket
 *       words zero again, a call that timed out included: a thread block that
 *       gives up still hands in its ticket for every segment it owned);
 *       calls sharing one workspace must not overlap.
 * dev_status  SPARDA_DEV_RANGE for skipped ids; SPARDA_DEV_TIMEOUT when a
 *       wait ran out, in which case the outputs of the call are not valid
 *       (the workspace is, for the next call).
 */
int sparda_sparse_attn_decode(const sparda_params *p, const void *Q, const void *K,
                              const void *V, long long bg_stride, long long blk_stride,
                              const int32_t *idx, int addr_mode, void *O, void *ws,
                              size_t ws_bytes, int32_t *dev_status, sparda_stream_t stream);

/*
 * sparda_sparse_attn_prefill -- every token of a query chunk attends over the
 * keys of its own block set (per token and group), causal, fp32 softmax.
 *   [p4 "The fourth projection", Algorithm 1 / Eq. 5]:
 *     O_l = attention(Q_l, K_l[B_l], V_l[B_l])   with all keys on the GPU
 * Q     bf16 [B][nq][Hq][d]; token i at position q_start + i <= T - 1 (with
 *       per-sequence lengths, at seq_len[b] - nq + i; q_start is then not used)
 * K, V  bf16, row (b,g,t) at base + (b*G+g)*bg_stride + t*tok_stride; this
 *       version needs tok_stride == d (else SPARDA_EUNSUPPORTED)
 * idx   int32 [B][nq][G][S] (as produced by sparda_forecast_select)
 * O     bf16 [B][nq][Hq][d]
 * ws    device workspace of sparda_workspace_size(SPARDA_OP_ATTN_PREFILL, p, nq, 0)
 *       bytes, zero-filled before its first use; calls sharing one workspace
 *       must not overlap.  ws and dev_status behave as for
 *       sparda_sparse_attn_decode (tickets restored after a timeout).
 */
int sparda_sparse_attn_prefill(const sparda_params *p, const void *Q, int nq, int q_start,
                               const void *K, const void *V, long long bg_stride,
                               long long tok_stride, const int32_t *idx, void *O, void *ws,
                               size_t ws_bytes, int32_t *dev_status, sparda_stream_t stream);

/*
 * sparda_sparse_attn_decode_noalloc -- sparda_sparse_attn_decode for callers
 * that cannot allocate device memory (code running under stream capture,
 * runtimes that own all device memory and hand kernels fixed buffers).  The
 * pages have no counterpart: this is a property of the library, not of the
 * method.  Arguments and results are those of sparda_sparse_attn_decode
 * without the workspace; the scratch lives in a fixed device array of
 * SPARDA_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until
 * the process exits.
 *  - shapes needing more scratch than that return SPARDA_EWORKSPACE;
 *  - every call shares the array, and each call clears the part that must
 *    start at zero: calls that may overlap on the device race and must not
 *    be issued;
 *  - the first call on a device looks up the array's device address with
 *    that device current; make it before any stream capture.
 * No cudaMalloc, cudaFree or other allocating routine is called.
 */
#define SPARDA_NOALLOC_SCRATCH_BYTES (8u << 20)
int sparda_sparse_attn_decode_noalloc(const sparda_params *p, const void *Q, const void *K,
                                      const void *V, long long bg_stride, long long blk_stride,
                                      const int32_t *idx, int addr_mode, void *O,
                                      int32_t *dev_status, sparda_stream_t stream);

/*
 * Device slot cache across decode steps -- fetch only what is new.
 *   [p4 "The fourth projection", Algorithm 2] fetches every layer's selected
 *   blocks from CPU pinned memory each step, and [p4 "What this doesn't
 *   fix"] notes that the host link bounds that transfer.  A block still
 *   selected at the next step need not cross the link again if it stays in
 *   the device slots.  The pages give no policy; these calls implement the
 *   plainest one.  Each (b,g) owns C slots (S <= C <= 4096) of one layer:
 *     cache     bf16 [B][G][C][2][blk][d] device (K block then V block)
 *     block_of  int32 [B][G][C] device: the block each slot holds, -1 empty
 *               (fill with -1 before the first step)
 *     hand      int32 [B][G] device: the clock position (0 before the first step)
 *   The state belongs to the caller; one layer's calls must not overlap.
 *
 * sparda_cache_plan -- for one step's lists idx [B][G][S] (device): an entry
 *   whose block some slot c holds is a hit (phys = c, fetch = 0); every other
 *   entry with a block id in [0, NB), in list order, takes the next slot past
 *   the hand that holds none of this step's blocks (phys = that slot,
 *   fetch = 1) and the hand moves one further.  Entries of -1 get phys = -1;
 *   ids >= NB are flagged SPARDA_DEV_RANGE.  block_of and hand are updated.
 *   phys, fetch: int32 [B][G][S] device (out).  C < S -> SPARDA_EINVAL.
 */
int sparda_cache_plan(const sparda_params *p, int C, const int32_t *idx, int32_t *block_of,
                      int32_t *hand, int32_t *phys, int32_t *fetch, int32_t *dev_status,
                      sparda_stream_t stream);

/*
 * sparda_prefetch_cached -- copy block idx[s] of the page-locked, mapped host
 *   buffer (layout and checks as for sparda_prefetch_blocks) into slot
 *   phys[s] of the cache, for every entry with fetch[s] != 0 (the misses of
 *   sparda_cache_plan); n_ctas as for sparda_prefetch_blocks.
 */
int sparda_prefetch_cached(const sparda_params *p, int C, const void *host_kv,
                           const int32_t *idx, const int32_t *phys, const int32_t *fetch,
                           void *cache, int n_ctas, int32_t *dev_status, sparda_stream_t stream);

/*
 * sparda_forecast_select_cached -- the decode selection (one query token)
 *   fused with the slot cache: the results of sparda_forecast_select (nq = 1)
 *   followed by sparda_cache_plan on the lists it wrote and
 *   sparda_prefetch_cached of the misses, from one launch.  The thread block
 *   that writes a (b,g)'s set plans that set against the pair's slots and
 *   copies its misses, so the next layer's attention waits on a single
 *   kernel, and the fetch of a pair starts as soon as its set is known.
 *   [p4 "The fourth projection", Algorithm 2]: select the next layer's
 *   blocks, then fetch them while the current layer computes.
 * F, nf, q_start, kc, idx, ws, ws_bytes  as for sparda_forecast_select with
 *       nq = 1 (the workspace of SPARDA_OP_SELECT with nq = 1)
 * C, block_of, hand, phys, fetch, cache  as for sparda_cache_plan and
 *       sparda_prefetch_cached (one layer's slots, updated in place)
 * host_kv  the page-locked, mapped host blocks, as for sparda_prefetch_cached
 * Block grid only; the cached state must not be shared with a call that
 * may overlap this one.  dev_status collects the flags of the three calls.
 */
int sparda_forecast_select_cached(const sparda_params *p, const void *F, int nf, int q_start,
                                  const void *kc, int32_t *idx, void *ws, size_t ws_bytes, int C,
                                  int32_t *block_of, int32_t *hand, int32_t *phys, int32_t *fetch,
                                  const void *host_kv, void *cache, int32_t *dev_status,
                                  sparda_stream_t stream);

/*
 * sparda_sparse_attn_decode_cached -- sparda_sparse_attn_decode reading list
 *   entry s of (b,g) from cache slot phys[b,g,s] (idx gives its block id for
 *   the causal mask).  A slot outside [0, C) is skipped and flagged
 *   SPARDA_DEV_RANGE.  ws as for sparda_sparse_attn_decode.
 */
int sparda_sparse_attn_decode_cached(const sparda_params *p, int C, const void *Q,
                                     const void *cache, const int32_t *idx, const int32_t *phys,
                                     void *O, void *ws, size_t ws_bytes, int32_t *dev_status,
                                     sparda_stream_t stream);

/* Bytes of device workspace an op needs for these shapes (0: none). nf is
 * the number of scoring vectors per group (select only). */
size_t sparda_workspace_size(int op, const sparda_params *p, int nq, int nf);

/* Human-readable name of a status code (static string). */
const char *sparda_status_string(int status);

/* Map a device status word to SPARDA_OK / SPARDA_ERANGE / SPARDA_ETIMEOUT. */
int sparda_status_from_device(int32_t word);

/* Library version, major*10000 + minor*100 + patch. */
int sparda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARDA_H_ */
