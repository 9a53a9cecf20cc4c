"""Thin Python binding of libsparda's C ABI (``include/sparda.h``).

Argument marshalling only: every step of the hot path runs in the CUDA
kernels of ``lib/libsparda.so``.  Tensors are torch tensors (device memory
and streams are PyTorch's); each function takes the same arguments, in the
same order, as the C entry point of the same name and raises ``SpardaError``
on a non-zero status.  There is no CPU fallback: if the library is missing,
loading it raises.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "lib", "libsparda.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "sparda.h")

SPARDA_OK = 0
SPARDA_EINVAL = -1
SPARDA_EUNSUPPORTED = -2
SPARDA_ECUDA = -3
SPARDA_ERANGE = -4
SPARDA_ETIMEOUT = -5
SPARDA_EWORKSPACE = -6

SPARDA_DEV_RANGE = 1
SPARDA_DEV_TIMEOUT = 2
SPARDA_DEV_LAYOUT = 4

SPARDA_OP_COMPRESS = 0
SPARDA_OP_SELECT = 1
SPARDA_OP_PREFETCH = 2
SPARDA_OP_ATTN_DECODE = 3
SPARDA_OP_ATTN_PREFILL = 4
SPARDA_OP_SELECT_WINDOWS = 5
SPARDA_OP_HEAD_SOFTMAX = 6
SPARDA_OP_HEAD_SOFTMAX_WINDOWS = 7

SPARDA_ADDR_LOGICAL = 0
SPARDA_ADDR_SLOT = 1
SPARDA_ADDR_PHYS = 2


class SpardaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__("%s failed: %s (%d)" % (fn, msg, status))
        self.status = status


class sparda_tuning(ctypes.Structure):
    _fields_ = [("select_chunk", ctypes.c_int), ("select_stream", ctypes.c_int),
                ("select_binned", ctypes.c_int), ("attn_ctas", ctypes.c_int),
                ("attn_stages", ctypes.c_int), ("attn_split_kv", ctypes.c_int),
                ("prefetch_ctas", ctypes.c_int), ("attn_prefill_per_token", ctypes.c_int),
                ("attn_wait_cycles", ctypes.c_longlong)]


class sparda_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("G", ctypes.c_int),
                ("d", ctypes.c_int), ("blk", ctypes.c_int), ("T", ctypes.c_int),
                ("k", ctypes.c_int), ("n_init", ctypes.c_int), ("n_local", ctypes.c_int),
                ("scale", ctypes.c_float), ("seq_len", ctypes.c_void_p),
                ("tune", ctypes.POINTER(sparda_tuning))]


def make_params(B, Hq, G, T, k, n_init=1, n_local=2, d=128, blk=64, scale=0.0,
                seq_len=None, tune=None) -> sparda_params:
    """seq_len: optional device int32 tensor [B] of per-sequence lengths (the
    caller keeps it alive while the params are in use).  tune: optional dict
    of sparda_tuning fields (launch choices; the rest stay 0, the library's
    own); the params keep the struct alive."""
    p = sparda_params(int(B), int(Hq), int(G), int(d), int(blk), int(T), int(k), int(n_init),
                      int(n_local), float(scale),
                      None if seq_len is None else seq_len.data_ptr())
    if tune:
        t = sparda_tuning(**{k_: int(v) for k_, v in tune.items()})
        p._tune_keep = t
        p.tune = ctypes.pointer(t)
    return p


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_LL = ctypes.c_longlong
_SZ = ctypes.c_size_t
_PP = ctypes.POINTER(sparda_params)

_SIGS = {
    "sparda_compress_keys": (_I, [_PP, _P, _LL, _LL, _P, _P, _P]),
    "sparda_forecast_select": (_I, [_PP, _P, _I, _I, _I, _P, _P, _P, _SZ, _P, _P]),
    "sparda_append_kv": (_I, [_PP, _I, _P, _P, _P, _P, _LL, _LL, _P, _P, _P]),
    "sparda_append_windows": (_I, [_PP, _I, _P, _LL, _LL, _I, _I, _P, _P, _P]),
    "sparda_compress_windows": (_I, [_PP, _P, _LL, _LL, _I, _I, _P, _P, _P]),
    "sparda_forecast_select_windows": (_I, [_PP, _P, _I, _I, _I, _P, _I, _I, _P, _P, _SZ, _P,
                                            _P]),
    "sparda_head_softmax_select": (_I, [_PP, _P, _I, _I, ctypes.c_float, _P, _P, _P, _SZ, _P,
                                        _P]),
    "sparda_head_softmax_select_windows": (_I, [_PP, _P, _I, _I, ctypes.c_float, _P, _I, _I, _P,
                                                _P, _SZ, _P, _P]),
    "sparda_prefetch_blocks": (_I, [_PP, _P, _P, _P, _I, _I, _P, _P]),
    "sparda_sparse_attn_decode": (_I, [_PP, _P, _P, _P, _LL, _LL, _P, _I, _P, _P, _SZ, _P, _P]),
    "sparda_sparse_attn_prefill": (_I, [_PP, _P, _I, _I, _P, _P, _LL, _LL, _P, _P, _P, _SZ, _P, _P]),
    "sparda_sparse_attn_decode_noalloc": (_I, [_PP, _P, _P, _P, _LL, _LL, _P, _I, _P, _P, _P]),
    "sparda_cache_plan": (_I, [_PP, _I, _P, _P, _P, _P, _P, _P, _P]),
    "sparda_prefetch_cached": (_I, [_PP, _I, _P, _P, _P, _P, _P, _I, _P, _P]),
    "sparda_forecast_select_cached": (_I, [_PP, _P, _I, _I, _P, _P, _P, _SZ, _I, _P, _P, _P,
                                           _P, _P, _P, _P, _P]),
    "sparda_sparse_attn_decode_cached": (_I, [_PP, _I, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "sparda_workspace_size": (_SZ, [_I, _PP, _I, _I]),
    "sparda_status_string": (ctypes.c_char_p, [_I]),
    "sparda_status_from_device": (_I, [ctypes.c_int32]),
    "sparda_version": (_I, []),
}


def lib() -> ctypes.CDLL:
    """Load libsparda.so (raises if it has not been built: no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError("libsparda.so not built (%s); run python -m "
                          "block_sparse_long_sparda_b200.build" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Entry points declared in include/sparda.h."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char \*)\s*(sparda_\w+)\s*\(", text, re.M)))


def _check(fn: str, st: int):
    if st != SPARDA_OK:
        raise SpardaError(fn, st, lib().sparda_status_string(st).decode())


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


# --------------------------------------------------------------------------
# entry points (same names and argument order as the C ABI)
# --------------------------------------------------------------------------

def sparda_compress_keys(p, K, bg_stride, tok_stride, kc_f32, kc_bf16, stream=None):
    _check("sparda_compress_keys",
           lib().sparda_compress_keys(ctypes.byref(p), _ptr(K), int(bg_stride), int(tok_stride),
                                      _ptr(kc_f32), _ptr(kc_bf16), _stream(stream)))


def sparda_append_kv(p, pos, K_new, V_new, K, V, bg_stride, blk_stride, kc_f32, kc_bf16,
                     stream=None):
    _check("sparda_append_kv",
           lib().sparda_append_kv(ctypes.byref(p), int(pos), _ptr(K_new), _ptr(V_new), _ptr(K),
                                  _ptr(V), int(bg_stride), int(blk_stride), _ptr(kc_f32),
                                  _ptr(kc_bf16), _stream(stream)))


def sparda_append_windows(p, pos, K, bg_stride, blk_stride, win, stride, kw_f32, kw_bf16,
                          stream=None):
    _check("sparda_append_windows",
           lib().sparda_append_windows(ctypes.byref(p), int(pos), _ptr(K), int(bg_stride),
                                       int(blk_stride), int(win), int(stride), _ptr(kw_f32),
                                       _ptr(kw_bf16), _stream(stream)))


def sparda_compress_windows(p, K, bg_stride, tok_stride, win, stride, kw_f32, kw_bf16,
                            stream=None):
    _check("sparda_compress_windows",
           lib().sparda_compress_windows(ctypes.byref(p), _ptr(K), int(bg_stride), int(tok_stride),
                                         int(win), int(stride), _ptr(kw_f32), _ptr(kw_bf16),
                                         _stream(stream)))


def sparda_forecast_select_windows(p, F, nq, nf, q_start, kw, win, stride, idx, ws,
                                   dev_status=None, stream=None):
    _check("sparda_forecast_select_windows",
           lib().sparda_forecast_select_windows(ctypes.byref(p), _ptr(F), int(nq), int(nf),
                                                int(q_start), _ptr(kw), int(win), int(stride),
                                                _ptr(idx), _ptr(ws), _nbytes(ws), _ptr(dev_status),
                                                _stream(stream)))


def sparda_forecast_select(p, F, nq, nf, q_start, kc, idx, ws, dev_status=None, stream=None):
    _check("sparda_forecast_select",
           lib().sparda_forecast_select(ctypes.byref(p), _ptr(F), int(nq), int(nf), int(q_start),
                                        _ptr(kc), _ptr(idx), _ptr(ws), _nbytes(ws),
                                        _ptr(dev_status), _stream(stream)))


def sparda_head_softmax_select(p, Q, nf, q_start, tau, kc, idx, ws, dev_status=None,
                               stream=None):
    _check("sparda_head_softmax_select",
           lib().sparda_head_softmax_select(ctypes.byref(p), _ptr(Q), int(nf), int(q_start),
                                            float(tau), _ptr(kc), _ptr(idx), _ptr(ws), _nbytes(ws),
                                            _ptr(dev_status), _stream(stream)))


def sparda_head_softmax_select_windows(p, Q, nf, q_start, tau, kw, win, stride, idx, ws,
                                       dev_status=None, stream=None):
    _check("sparda_head_softmax_select_windows",
           lib().sparda_head_softmax_select_windows(ctypes.byref(p), _ptr(Q), int(nf),
                                                    int(q_start), float(tau), _ptr(kw), int(win),
                                                    int(stride), _ptr(idx), _ptr(ws), _nbytes(ws),
                                                    _ptr(dev_status), _stream(stream)))


def sparda_prefetch_blocks(p, host_kv, idx, slots, skip_resident, n_ctas=0, dev_status=None,
                           stream=None):
    _check("sparda_prefetch_blocks",
           lib().sparda_prefetch_blocks(ctypes.byref(p), _ptr(host_kv), _ptr(idx), _ptr(slots),
                                        int(bool(skip_resident)), int(n_ctas), _ptr(dev_status),
                                        _stream(stream)))


def sparda_sparse_attn_decode(p, Q, K, V, bg_stride, blk_stride, idx, addr_mode, O, ws,
                              dev_status=None, stream=None):
    _check("sparda_sparse_attn_decode",
           lib().sparda_sparse_attn_decode(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V),
                                           int(bg_stride), int(blk_stride), _ptr(idx),
                                           int(addr_mode), _ptr(O), _ptr(ws), _nbytes(ws),
                                           _ptr(dev_status), _stream(stream)))


def sparda_sparse_attn_prefill(p, Q, nq, q_start, K, V, bg_stride, tok_stride, idx, O, ws,
                               dev_status=None, stream=None):
    _check("sparda_sparse_attn_prefill",
           lib().sparda_sparse_attn_prefill(ctypes.byref(p), _ptr(Q), int(nq), int(q_start),
                                            _ptr(K), _ptr(V), int(bg_stride), int(tok_stride),
                                            _ptr(idx), _ptr(O), _ptr(ws), _nbytes(ws),
                                            _ptr(dev_status), _stream(stream)))


def sparda_sparse_attn_decode_noalloc(p, Q, K, V, bg_stride, blk_stride, idx, addr_mode, O,
                                      dev_status=None, stream=None):
    """Decode attention for callers that cannot allocate device memory: the
    scratch is a fixed device array inside the library (see include/sparda.h
    for its size and the rule that calls must not overlap on the device)."""
    _check("sparda_sparse_attn_decode_noalloc",
           lib().sparda_sparse_attn_decode_noalloc(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V),
                                                   int(bg_stride), int(blk_stride), _ptr(idx),
                                                   int(addr_mode), _ptr(O), _ptr(dev_status),
                                                   _stream(stream)))


NOALLOC_SCRATCH_BYTES = 8 << 20


def sparda_cache_plan(p, C, idx, block_of, hand, phys, fetch, dev_status=None, stream=None):
    _check("sparda_cache_plan",
           lib().sparda_cache_plan(ctypes.byref(p), int(C), _ptr(idx), _ptr(block_of), _ptr(hand),
                                   _ptr(phys), _ptr(fetch), _ptr(dev_status), _stream(stream)))


def sparda_prefetch_cached(p, C, host_kv, idx, phys, fetch, cache, n_ctas=0, dev_status=None,
                           stream=None):
    _check("sparda_prefetch_cached",
           lib().sparda_prefetch_cached(ctypes.byref(p), int(C), _ptr(host_kv), _ptr(idx),
                                        _ptr(phys), _ptr(fetch), _ptr(cache), int(n_ctas),
                                        _ptr(dev_status), _stream(stream)))


def sparda_forecast_select_cached(p, F, nf, q_start, kc, idx, ws, C, block_of, hand, phys,
                                  fetch, host_kv, cache, dev_status=None, stream=None):
    _check("sparda_forecast_select_cached",
           lib().sparda_forecast_select_cached(ctypes.byref(p), _ptr(F), int(nf), int(q_start),
                                               _ptr(kc), _ptr(idx), _ptr(ws), _nbytes(ws), int(C),
                                               _ptr(block_of), _ptr(hand), _ptr(phys), _ptr(fetch),
                                               _ptr(host_kv), _ptr(cache), _ptr(dev_status),
                                               _stream(stream)))


def sparda_sparse_attn_decode_cached(p, C, Q, cache, idx, phys, O, ws, dev_status=None,
                                     stream=None):
    _check("sparda_sparse_attn_decode_cached",
           lib().sparda_sparse_attn_decode_cached(ctypes.byref(p), int(C), _ptr(Q), _ptr(cache),
                                                  _ptr(idx), _ptr(phys), _ptr(O), _ptr(ws),
                                                  _nbytes(ws), _ptr(dev_status), _stream(stream)))


def sparda_workspace_size(op, p, nq=1, nf=1) -> int:
    return int(lib().sparda_workspace_size(int(op), ctypes.byref(p), int(nq), int(nf)))


def sparda_status_string(status) -> str:
    return lib().sparda_status_string(int(status)).decode()


def sparda_status_from_device(word) -> int:
    return int(lib().sparda_status_from_device(int(word)))


def sparda_version() -> int:
    return int(lib().sparda_version())


# --------------------------------------------------------------------------
# allocation helpers (plumbing: torch owns the memory)
# --------------------------------------------------------------------------

def workspace(op, p, nq=1, nf=1, device="cuda"):
    """Zero-filled device workspace for an op (None when the op needs none)."""
    import torch
    n = sparda_workspace_size(op, p, nq, nf)
    if n == 0:
        return None
    return torch.zeros((n + 15) // 16 * 16, dtype=torch.uint8, device=device)
