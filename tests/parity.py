"""Helpers shared by the GPU parity tests: host<->device marshalling of bf16
bit arrays and the comparison rules (spec tolerances).

Comparison rules
- compressed keys: fp32 output within 1e-3 max abs of the fp64 oracle; the
  bf16 output equals the oracle's one-step rounding except for rare double
  rounding (>= 99.99% identical, never more than one unit in the last place);
- block sets: bit-exact wherever the oracle's k-th and (k+1)-th scores differ
  by more than 1e-3 relative; inside that band a set is valid when it has a
  set's structure (the oracle's size, -1 padding, initial and local blocks;
  ascending, causal, no repeats), keeps every block scoring clearly above
  the band and adds only blocks inside it;
- attention outputs: max abs error <= 1e-2 and relative L2 error <= 5e-3.
"""
from __future__ import annotations

import numpy as np
import torch

from block_sparse_long_sparda_b200 import workloads as W

ATTN_MAX_ABS = 1e-2
ATTN_REL_L2 = 5e-3
KC_MAX_ABS = 1e-3
TIE_REL = 1e-3


GUARD_BYTES = 4096
GUARD_BYTE = 0xA5


class Guarded:
    """A device output buffer with GUARD_BYTES of sentinel bytes before and
    after it, to catch writes outside the buffer (compute-sanitizer is not
    available on the GPU pool, so parity tests check the neighbourhood of
    their outputs instead).  ``t`` is the buffer (16-byte aligned, as the
    library needs); ``check()`` asserts that both guards are untouched."""

    def __init__(self, shape, dtype, fill=None, device="cuda"):
        shape = tuple(int(x) for x in shape)
        n = int(np.prod(shape)) if shape else 1
        esize = torch.empty(0, dtype=dtype).element_size()
        self.g = GUARD_BYTES // esize
        self.raw = torch.empty(self.g + n + self.g, dtype=dtype, device=device)
        self.raw.view(torch.uint8).fill_(GUARD_BYTE)
        self.t = self.raw[self.g:self.g + n].view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, what=""):
        torch.cuda.synchronize()
        b = self.raw.view(torch.uint8)
        gb = self.g * self.raw.element_size()
        head, tail = b[:gb], b[b.numel() - gb:]
        bad_h = int((head != GUARD_BYTE).sum().item())
        bad_t = int((tail != GUARD_BYTE).sum().item())
        assert bad_h == 0 and bad_t == 0, \
            "%s: %d bytes written before and %d after the output buffer" % (what, bad_h, bad_t)
        return self.t


def guarded_workspace(op, p, nq=1, nf=1):
    """A zero-filled workspace for an op inside guard regions (None when the
    op needs none)."""
    from block_sparse_long_sparda_b200 import abi
    n = abi.sparda_workspace_size(op, p, nq, nf)
    if n == 0:
        return None
    return Guarded(((n + 15) // 16 * 16,), torch.uint8, fill=0)


def dev_bf16(a: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bits (numpy) -> torch.bfloat16 on the device."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def host_bits(t: torch.Tensor) -> np.ndarray:
    """torch.bfloat16 (any device) -> uint16 numpy bits."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_f64(bits: np.ndarray) -> np.ndarray:
    return W.bf16_bits_to_f32(bits).astype(np.float64)


def check_attention(gpu_bits: np.ndarray, oracle_f64: np.ndarray, what: str = ""):
    g = bf16_f64(gpu_bits)
    o = np.asarray(oracle_f64, np.float64)
    assert g.shape == o.shape, (g.shape, o.shape)
    assert np.all(np.isfinite(g)), what + ": non-finite output"
    err = np.abs(g - o)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30))
    assert max_abs <= ATTN_MAX_ABS, "%s: max abs %.3e" % (what, max_abs)
    assert rel <= ATTN_REL_L2, "%s: rel L2 %.3e" % (what, rel)
    return max_abs, rel


def check_compressed(kc32: np.ndarray, kc16: np.ndarray, ora64: np.ndarray, ora16: np.ndarray):
    err = float(np.abs(kc32.astype(np.float64) - ora64).max())
    assert err <= KC_MAX_ABS, "fp32 Kc max abs %.3e" % err
    same = np.mean(kc16 == ora16)
    assert same >= 0.9999, "bf16 Kc identical fraction %.6f" % same
    diff = np.abs(kc16.astype(np.int32) - ora16.astype(np.int32))
    assert diff.max() <= 1, "bf16 Kc differs by more than one ulp"
    return err, same


def scores_f64(F_bits: np.ndarray, kc_bits: np.ndarray) -> np.ndarray:
    """Summed dot products in fp64 for the band rule.
    F [B][nq][G][nf][d], kc [B][G][NB][d] -> [B][nq][G][NB]."""
    F = bf16_f64(F_bits).sum(axis=3)                      # sum over the nf vectors
    kc = bf16_f64(kc_bits)
    return np.einsum("bqgd,bgnd->bqgn", F, kc)


def candidate_range(pos, n_init, n_local, blk=64):
    """(c, lo, hi): the query's own block c and its candidate blocks [lo, hi)
    -- the causal blocks that are neither initial nor local (readings R1 and
    R2: local = [max(0, c - n_local + 1), c], initial = [0, n_init) minus the
    local ones)."""
    c = int(pos) // blk
    local_lo = max(0, c - n_local + 1)
    return c, n_init, max(local_lo, n_init)


def check_sets(gpu_idx: np.ndarray, ora_idx: np.ndarray, kth: np.ndarray, kth1: np.ndarray,
               scores: np.ndarray | None, what: str = "", *, q_pos, n_init: int, n_local: int,
               blk: int = 64):
    """gpu_idx/ora_idx [B][nq][G][S]; kth/kth1 [B][nq][G]; scores [B][nq][G][NB];
    q_pos: each query's position, a scalar or an array broadcastable to [B][nq].

    Where the oracle's k-th and (k+1)-th scores differ by more than TIE_REL
    relative the sets must be identical.  Inside that band another set is
    valid only if it has the structure of one: the same number of entries
    with the -1 padding at the same positions, ascending and without
    repeats, every id causal, exactly the oracle's initial and local blocks
    (so as many candidates as the oracle's), no block scoring clearly above
    the band dropped and no block scoring clearly below it added."""
    assert gpu_idx.shape == ora_idx.shape, (gpu_idx.shape, ora_idx.shape)
    qp = np.broadcast_to(np.asarray(q_pos), gpu_idx.shape[:2])
    exact = bitexact = 0
    for pos in np.ndindex(*gpu_idx.shape[:3]):
        g, o = gpu_idx[pos], ora_idx[pos]
        a, b = kth[pos], kth1[pos]
        clear = not np.isfinite(b) or not np.isfinite(a) or abs(a - b) > TIE_REL * abs(a)
        if np.array_equal(g, o):
            bitexact += 1
            exact += clear
            continue
        assert not clear, "%s %s: sets differ with a clear k-th gap\n gpu %s\n ora %s" % (what, pos, g, o)
        assert scores is not None, "%s %s: near tie but no scores to check the band" % (what, pos)
        assert np.array_equal(g < 0, o < 0), \
            "%s %s: entries or -1 padding differ from the oracle's\n gpu %s\n ora %s" % (what, pos, g, o)
        valid = g[g >= 0]
        assert len(set(valid.tolist())) == len(valid), "%s %s: duplicate ids" % (what, pos)
        assert np.all(np.diff(valid) > 0), "%s %s: not ascending" % (what, pos)
        c, lo, hi = candidate_range(qp[pos[:2]], n_init, n_local, blk)
        assert np.all(valid <= c), "%s %s: a block after the query's own" % (what, pos)
        gs, os_ = set(valid.tolist()), set(o[o >= 0].tolist())
        fixed_g = {j for j in gs if not lo <= j < hi}
        fixed_o = {j for j in os_ if not lo <= j < hi}
        assert fixed_g == fixed_o, "%s %s: initial/local blocks %s, oracle %s" % (
            what, pos, sorted(fixed_g), sorted(fixed_o))
        hi_band = a + TIE_REL * abs(a)
        lo_band = a - TIE_REL * abs(a)
        sc = scores[pos]
        for j in os_ - gs:
            assert sc[j] <= hi_band, "%s %s: dropped block %d scoring above the band" % (what, pos, j)
        for j in gs - os_:
            assert sc[j] >= lo_band, "%s %s: added block %d scoring below the band" % (what, pos, j)
    return bitexact


def pooled_scores_f64(F_bits, kw_bits, NB):
    """fp64 block scores of the window grid for the band rule: the best of
    the windows 4j, 4j+1, 4j+2 that exist.  -> [B][nq][G][NB]"""
    ws = scores_f64(F_bits, kw_bits)                 # [B][nq][G][NW]
    NW = ws.shape[-1]
    out = np.full(ws.shape[:3] + (NB,), -np.inf)
    for j in range(NB):
        cols = [w for w in (4 * j, 4 * j + 1, 4 * j + 2) if w < NW]
        if cols:
            out[..., j] = ws[..., cols].max(axis=-1)
    return out
