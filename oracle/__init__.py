"""Plain fp64 CPU oracle for the SparDA hot path -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and
this package imports nothing from it: the two share no code.

The arithmetic lives in ``sparda_oracle.c`` (plain C, double precision, loops
written straight from the definitions); this module only compiles it with gcc
and marshals numpy arrays.  bf16 tensors are passed as ``uint16`` arrays of
their raw bits and decoded exactly inside the C code.

Sources: "SparDA: a fourth projection that lets sparse attention prefetch its
own KV cache" (ai.thesatyajit.com/articles/sparda) -- section "The problem
InfLLM-V2 leaves on the table" (eq. B_l(i)), section "The fourth projection"
(Eq. 3-5, Algorithms 1 and 2), section "One Forecast head per GQA group"
(Forecast indexer versus the multi-head baseline selector); and
deepresearch2agi.pages.dev/sparda_sparse_decoupled_attention, section
"架构细节" (mean-compressed keys).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sparda_oracle.c")
_LIB = os.path.join(_HERE, "libsparda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libsparda_oracle.so`` (gcc, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-D_DEFAULT_SOURCE", "-fPIC", "-shared",
             "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        LL = ctypes.c_longlong
        D = ctypes.c_double
        lib.oracle_double_to_bf16.argtypes = [D]
        lib.oracle_double_to_bf16.restype = ctypes.c_uint16
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = D
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = I
        lib.oracle_compress_keys.argtypes = [I, I, I, I, I, P, LL, LL, P, P]
        lib.oracle_compress_keys.restype = None
        lib.oracle_select.argtypes = [I, I, I, I, I, I, I, I, I, I, I, P, P, P, P, P]
        lib.oracle_select.restype = None
        lib.oracle_gather_blocks.argtypes = [I, I, I, I, I, I, I, I, I, I, P, P, P]
        lib.oracle_gather_blocks.restype = None
        lib.oracle_window_count.argtypes = [I, I, I]
        lib.oracle_window_count.restype = I
        lib.oracle_compress_windows.argtypes = [I, I, I, I, I, I, P, LL, LL, P, P]
        lib.oracle_compress_windows.restype = None
        lib.oracle_select_windows.argtypes = [I, I, I, I, I, I, I, I, I, I, I, I, I, P, P, P, P, P]
        lib.oracle_select_windows.restype = None
        lib.oracle_select_head_softmax.argtypes = [I, I, I, I, I, I, I, I, I, I, I, I, I, D,
                                                   P, P, P, P, P, P]
        lib.oracle_select_head_softmax.restype = None
        lib.oracle_cache_plan.argtypes = [I, I, I, I, I, P, P, P, P, P]
        lib.oracle_cache_plan.restype = I
        lib.oracle_gather_cached.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P]
        lib.oracle_gather_cached.restype = None
        lib.oracle_sparse_attention.argtypes = [I, I, I, I, I, I, I, I, D, P, P, P, LL, LL, P, I, P]
        lib.oracle_sparse_attention.restype = None
        lib.oracle_dense_causal_attention.argtypes = [I, I, I, I, I, I, I, D, P, P, P, P]
        lib.oracle_dense_causal_attention.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as uint16 arrays of raw bits, got %s" % a.dtype)
    return a


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def double_to_bf16(x: float) -> int:
    """Round one double to bf16 bits, to nearest, ties to even (one rounding)."""
    return int(_load().oracle_double_to_bf16(float(x)))


def bf16_to_double(bits: int) -> float:
    return float(_load().oracle_bf16_to_double(int(bits)))


def compress_keys(K: np.ndarray, blk: int = 64, shape=None, strides=None):
    """Mean-pooled compressed keys.

    K: uint16 [B][G][T][d].  Returns (kc_f64 [B][G][NB][d], kc_bf16 [B][G][NB][d]).
    With ``shape=(B, G, T, d)`` and ``strides=(bg_stride, tok_stride)`` (elements)
    K may be any buffer holding row (b,g,t) at (b*G+g)*bg_stride + t*tok_stride.
    """
    K = _u16(K)
    if shape is None:
        B, G, T, d = K.shape
        bg_stride, tok_stride = T * d, d
    else:
        B, G, T, d = shape
        bg_stride, tok_stride = strides
        assert (B * G - 1) * bg_stride + (T - 1) * tok_stride + d <= K.size
    NB = (T + blk - 1) // blk
    kc = np.empty((B, G, NB, d), np.float64)
    kcb = np.empty((B, G, NB, d), np.uint16)
    _load().oracle_compress_keys(B, G, T, d, blk, _ptr(K), bg_stride, tok_stride, _ptr(kc),
                                 _ptr(kcb))
    return kc, kcb


def window_count(T: int, win: int = 32, stride: int = 16) -> int:
    return int(_load().oracle_window_count(int(T), int(win), int(stride)))


def compress_windows(K: np.ndarray, win: int = 32, stride: int = 16):
    """Window-grid compressed keys: mean of positions [w*stride, w*stride+win).

    K: uint16 [B][G][T][d].  Returns (kw_f64 [B][G][NW][d], kw_bf16 [B][G][NW][d])."""
    K = _u16(K)
    B, G, T, d = K.shape
    NW = window_count(T, win, stride)
    kw = np.empty((B, G, NW, d), np.float64)
    kwb = np.empty((B, G, NW, d), np.uint16)
    _load().oracle_compress_windows(B, G, T, d, win, stride, _ptr(K), T * d, d, _ptr(kw), _ptr(kwb))
    return kw, kwb


def select_windows(F: np.ndarray, kw: np.ndarray, T: int, k: int, n_init: int, n_local: int,
                   q_start: int, blk: int = 64, win: int = 32, stride: int = 16):
    """Block sets from window-grid keys: a block's score is the largest score
    of the windows inside it.  F [B][nq][G][nf][d]; kw [B][G][NW][d].
    Returns (idx [B][nq][G][S], kth, kth1) as select()."""
    F = _u16(F)
    kw = _u16(kw)
    B, nq, G, nf, d = F.shape
    assert kw.shape[:2] == (B, G) and kw.shape[2] == window_count(T, win, stride)
    S = k + n_init + n_local
    idx = np.empty((B, nq, G, S), np.int32)
    kth = np.empty((B, nq, G), np.float64)
    kth1 = np.empty((B, nq, G), np.float64)
    _load().oracle_select_windows(B, nq, G, nf, d, blk, win, stride, T, k, n_init, n_local,
                                  q_start, _ptr(F), _ptr(kw), _ptr(idx), _ptr(kth), _ptr(kth1))
    return idx, kth, kth1


def select(F: np.ndarray, kc: np.ndarray, k: int, n_init: int, n_local: int, q_start: int,
           blk: int = 64):
    """Block sets init U local U top-k(F . Kc^T).

    F:  uint16 [B][nq][G][nf][d] (nf = 1 for the Forecast indexer, nf = query heads
        per group for the baseline multi-head selector, whose scores are summed).
    kc: uint16 [B][G][NB][d].
    Query token i sits at position q_start + i.
    Returns (idx int32 [B][nq][G][S], kth [B][nq][G], kth1 [B][nq][G]).
    """
    F = _u16(F)
    kc = _u16(kc)
    B, nq, G, nf, d = F.shape
    NB = kc.shape[2]
    assert kc.shape == (B, G, NB, d)
    last = q_start + nq - 1
    if last // blk >= NB:
        raise ValueError("query position %d needs block %d but Kc has %d blocks" % (last, last // blk, NB))
    S = k + n_init + n_local
    idx = np.empty((B, nq, G, S), np.int32)
    kth = np.empty((B, nq, G), np.float64)
    kth1 = np.empty((B, nq, G), np.float64)
    _load().oracle_select(B, nq, G, nf, d, blk, NB, k, n_init, n_local, q_start,
                          _ptr(F), _ptr(kc), _ptr(idx), _ptr(kth), _ptr(kth1))
    return idx, kth, kth1


def select_head_softmax(Q: np.ndarray, kc: np.ndarray, T: int, k: int, n_init: int,
                        n_local: int, q_start: int, tau: float, windows: bool = False,
                        blk: int = 64, win: int = 32, stride: int = 16):
    """The original selector's per-head softmax form ("Training: distilling
    the selector you already have", Eq. 6): block weights
    S = sum over the group's query heads of softmax(Q_h . Kc^T / tau) over the
    key rows the query sees, max-pooled to blocks on the window grid; the
    set is init U top-k(S) U local.

    Q:  uint16 [B][G][nf][d] (the decode query's heads by group).
    kc: uint16 [B][G][NB][d] block keys, or [B][G][NW][d] window keys.
    Returns (idx [B][G][S], kth [B][G], kth1 [B][G], wblk [B][G][NB]).
    """
    Q = _u16(Q)
    kc = _u16(kc)
    B, G, nf, d = Q.shape
    NR = kc.shape[2]
    assert kc.shape == (B, G, NR, d)
    NB = (T + blk - 1) // blk
    if windows:
        assert NR == window_count(T, win, stride)
    else:
        assert NR == NB
    S = k + n_init + n_local
    idx = np.empty((B, G, S), np.int32)
    kth = np.empty((B, G), np.float64)
    kth1 = np.empty((B, G), np.float64)
    wblk = np.empty((B, G, NB), np.float64)
    _load().oracle_select_head_softmax(B, G, nf, d, blk, win if windows else 0, stride, T, NR,
                                       k, n_init, n_local, q_start, float(tau), _ptr(Q), _ptr(kc),
                                       _ptr(idx), _ptr(kth), _ptr(kth1), _ptr(wblk))
    return idx, kth, kth1, wblk


def gather_blocks(host_kv: np.ndarray, idx: np.ndarray, pos: int, n_init: int, n_local: int,
                  skip_resident: bool, slots: np.ndarray | None = None) -> np.ndarray:
    """Byte copy of the selected blocks into slots.

    host_kv: uint16 [B][G][NB][2][blk][d]; idx int32 [B][G][S].
    Returns slots uint16 [B][G][S][2][blk][d] (entries not copied keep the
    contents of ``slots`` if given, else zero).
    """
    host_kv = _u16(host_kv)
    B, G, NB, two, blk, d = host_kv.shape
    idx = np.ascontiguousarray(idx, np.int32)
    S = idx.shape[-1]
    if slots is None:
        slots = np.zeros((B, G, S, 2, blk, d), np.uint16)
    else:
        slots = np.ascontiguousarray(slots.copy())
    _load().oracle_gather_blocks(B, G, NB, S, blk, d, pos, n_init, n_local, int(skip_resident),
                                 _ptr(host_kv), _ptr(idx), _ptr(slots))
    return slots


def cache_plan(idx: np.ndarray, block_of: np.ndarray, hand: np.ndarray, NB: int):
    """One step of the device slot cache (see oracle_cache_plan).

    idx int32 [B][G][S]; block_of int32 [B][G][C] and hand int32 [B][G] are the
    cache state before the step.  Returns (phys, fetch, block_of', hand')."""
    idx = np.ascontiguousarray(idx, np.int32)
    blk = np.ascontiguousarray(block_of, np.int32).copy()
    hd = np.ascontiguousarray(hand, np.int32).copy()
    B, G, S = idx.shape
    C = blk.shape[2]
    assert blk.shape == (B, G, C) and hd.shape == (B, G)
    phys = np.empty((B, G, S), np.int32)
    fetch = np.empty((B, G, S), np.int32)
    rc = _load().oracle_cache_plan(B, G, S, C, int(NB), _ptr(idx), _ptr(blk), _ptr(hd),
                                   _ptr(phys), _ptr(fetch))
    if rc != 0:
        raise ValueError("cache_plan needs C >= S (C=%d, S=%d)" % (C, S))
    return phys, fetch, blk, hd


def gather_cached(host_kv: np.ndarray, idx: np.ndarray, phys: np.ndarray, fetch: np.ndarray,
                  cache: np.ndarray) -> np.ndarray:
    """Copy the fetched blocks into their slots.  host_kv [B][G][NB][2][blk][d],
    cache [B][G][C][2][blk][d] (returned as an updated copy)."""
    host_kv = _u16(host_kv)
    B, G, NB, two, blk, d = host_kv.shape
    cache = np.ascontiguousarray(_u16(cache).copy())
    C = cache.shape[2]
    idx = np.ascontiguousarray(idx, np.int32)
    S = idx.shape[-1]
    _load().oracle_gather_cached(B, G, NB, S, C, blk, d, _ptr(host_kv), _ptr(idx),
                                 _ptr(np.ascontiguousarray(phys, np.int32)),
                                 _ptr(np.ascontiguousarray(fetch, np.int32)), _ptr(cache))
    return cache


def sparse_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray, q_start: int,
                     T: int, blk: int = 64, scale: float = 0.0, bg_stride: int | None = None,
                     blk_stride: int | None = None, G: int | None = None) -> np.ndarray:
    """Attention over the keys of each query's block set (fp64 result).

    Q: uint16 [B][nq][Hq][d]; idx int32 [B][nq][G][S].
    K/V: uint16, either [B][G][T][d] (strides derived) or any buffer with the
    row of token t of (b,g) at (b*G+g)*bg_stride + (t//blk)*blk_stride + (t%blk)*d.
    """
    Q = _u16(Q)
    K = _u16(K)
    V = _u16(V)
    B, nq, Hq, d = Q.shape
    idx = np.ascontiguousarray(idx, np.int32)
    if G is None:
        G = idx.shape[2]
    S = idx.shape[3]
    if bg_stride is None:
        assert K.ndim == 4 and K.shape[0] == B and K.shape[1] == G and K.shape[3] == d
        bg_stride = K.shape[2] * d
        blk_stride = blk * d
    O = np.empty((B, nq, Hq, d), np.float64)
    _load().oracle_sparse_attention(B, nq, Hq, G, d, blk, T, q_start, float(scale), _ptr(Q),
                                    _ptr(K), _ptr(V), int(bg_stride), int(blk_stride), _ptr(idx),
                                    S, _ptr(O))
    return O


def dense_causal_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, q_start: int,
                           scale: float = 0.0) -> np.ndarray:
    """Textbook causal softmax attention.  Q [B][nq][Hq][d]; K/V [B][G][T][d]."""
    Q = _u16(Q)
    K = _u16(K)
    V = _u16(V)
    B, nq, Hq, d = Q.shape
    G, T = K.shape[1], K.shape[2]
    O = np.empty((B, nq, Hq, d), np.float64)
    _load().oracle_dense_causal_attention(B, nq, Hq, G, d, T, q_start, float(scale), _ptr(Q),
                                          _ptr(K), _ptr(V), _ptr(O))
    return O
