// noalloc.cu -- decode attention for callers that cannot allocate device
// memory.
//
// Some callers cannot call cudaMalloc: code running while a CUDA graph is
// being captured, allocators that forbid allocation on the decode path,
// runtimes that own every byte of device memory and hand kernels fixed
// buffers only.  For them this file keeps the scratch that the decode
// attention kernel needs (its per-segment partial outputs and the tickets
// that decide which CTA combines them) in a fixed, file-scope device array
// instead of a caller-provided workspace.  The caller still passes every
// input and output buffer.
//
// Costs and limits, stated once:
//  - the array holds SPARDA_NOALLOC_SCRATCH_BYTES (8 MiB) on every GPU that
//    loads the library, until the process exits;
//  - shapes whose scratch would exceed it are rejected (SPARDA_EWORKSPACE);
//  - all calls share the one array: calls that may overlap on the GPU (on
//    different streams, or from different host threads without ordering)
//    race on it and must not be issued;
//  - the array keeps the previous call's contents, so each call clears the
//    ticket words that must start at zero before its kernel runs;
//  - the first call in a CUDA context (per device, and again after a device
//    reset or a new primary context, which reload the module and move the
//    array) resolves the array's device address with cudaGetSymbolAddress,
//    that device current; make that first call before any stream capture.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/sparda.h"
#include "common.cuh"
#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[SPARDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_lock;
struct ScratchAddr {
  void *ctx;   // the context the address was resolved in
  void *ptr;   // the array's device address there
};
ScratchAddr g_scratch[kMaxDevices] = {};

// Device address of the scratch array in the current context (resolved once
// per device and context).  In host code the array's name only stands in for
// it.
int scratch_for_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return SPARDA_ECUDA;
  }
  void *ctx = sparda::current_context();
  std::lock_guard<std::mutex> guard(g_setup_lock);
  ScratchAddr &e = g_scratch[dev];
  if (!e.ptr || !ctx || e.ctx != ctx) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      e = ScratchAddr{};
      return SPARDA_ECUDA;
    }
    // cudaGetSymbolAddress makes the primary context current if none was
    e = ScratchAddr{ctx ? ctx : sparda::current_context(), p};
  }
  *out = e.ptr;
  return SPARDA_OK;
}

}  // namespace

extern "C" int sparda_sparse_attn_decode_noalloc(const sparda_params *p, const void *Q,
                                                 const void *K, const void *V, long long bg_stride,
                                                 long long blk_stride, const int32_t *idx,
                                                 int addr_mode, void *O, int32_t *dev_status,
                                                 sparda_stream_t stream) {
  using namespace sparda;
  // the same argument rules as sparda_sparse_attn_decode
  const int pst = check_params(p);
  if (pst != SPARDA_OK) return pst;
  if (addr_mode != SPARDA_ADDR_LOGICAL && addr_mode != SPARDA_ADDR_SLOT) return SPARDA_EINVAL;
  if (p->B == 0) return SPARDA_OK;
  if (!Q || !K || !V || !idx || !O) return SPARDA_EINVAL;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) |
                        reinterpret_cast<uintptr_t>(V) | reinterpret_cast<uintptr_t>(idx) |
                        reinterpret_cast<uintptr_t>(O);
  if (mis & 15u) return SPARDA_EINVAL;
  if (bg_stride <= 0 || blk_stride < (long long)kBlk * kD || bg_stride % 8 || blk_stride % 8)
    return SPARDA_EINVAL;

  const DecodePlan pl = plan_decode(*p);
  if (pl.ws_bytes > (size_t)SPARDA_NOALLOC_SCRATCH_BYTES) return SPARDA_EWORKSPACE;

  void *scratch = nullptr;
  const int st = scratch_for_current_device(&scratch);
  if (st != SPARDA_OK) return st;

  // the ticket words (where the plan puts them) must start at zero
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(static_cast<char *>(scratch) + pl.ws_ticket_off, 0, pl.ws_ticket_bytes, s) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return SPARDA_ECUDA;
  }
  const cudaError_t e = launch_attn_decode(*p, pl, static_cast<const uint16_t *>(Q),
                                           static_cast<const uint16_t *>(K),
                                           static_cast<const uint16_t *>(V), bg_stride, blk_stride,
                                           idx, addr_mode, static_cast<uint16_t *>(O), scratch,
                                           dev_status, s);
  return e == cudaSuccess ? SPARDA_OK : SPARDA_ECUDA;
}
