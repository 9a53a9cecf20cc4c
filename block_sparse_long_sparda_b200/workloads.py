"""Seeded synthetic workloads for the SparDA hot path.

This module only draws random inputs and describes workload shapes.  It holds
none of the method's arithmetic (no pooling, scoring, ranking or attention),
so both the CUDA path and the CPU oracle may consume what it produces.

All bf16 tensors are produced as raw bits (``uint16``): values are drawn in
fp32 (numpy PCG64, or torch's Philox generator for the multi-GB host KV of the
decode loop) and rounded to bf16 to nearest, ties to even.

The shapes stand in for the pages' own workloads (8B block-sparse models at
128K context, batch 4 prefill and batch 16+ decode; the article "SparDA: a
fourth projection that lets sparse attention prefetch its own KV cache",
section "Three speedups, three different baselines"), which use trained
weights we do not have: every tensor
here is N(0, 1) noise with the structure the workload names (planted hot
blocks for the recall case).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hq: int
    G: int
    k: int
    seed: int
    d: int = 128
    blk: int = 64
    n_init: int = 1
    n_local: int = 2
    nq: int = 1            # query tokens per sequence (1 = decode)
    layers: int = 1        # decode loop depth
    planted: int = 0       # hot blocks planted per (b, g)
    min_len: int = 0       # > 0: per-sequence lengths drawn uniformly in [min_len, T]
    windows: int = 0       # 1: selection on the window grid (32 tokens, stride 16)
    note: str = ""

    @property
    def NB(self) -> int:
        return (self.T + self.blk - 1) // self.blk

    @property
    def S(self) -> int:
        return self.k + self.n_init + self.n_local

    @property
    def r(self) -> int:
        return self.Hq // self.G

    @property
    def q_start(self) -> int:
        return self.T - self.nq


WORKLOADS = {
    "decode_b1_t4k": Workload(
        "decode_b1_t4k", B=1, T=4096, Hq=16, G=2, k=4, seed=1001,
        note="decode step, one layer, all KV in HBM"),
    "decode_b4_t32k_planted": Workload(
        "decode_b4_t32k_planted", B=4, T=32768, Hq=32, G=8, k=32, planted=16, seed=1002,
        note="decode step, one layer, 16 hot blocks per group shifted toward the Forecast"),
    "decode_loop_b16_t128k": Workload(
        "decode_loop_b16_t128k", B=16, T=131072, Hq=32, G=8, k=64, layers=4, seed=1003,
        note="4-layer decode loop, KV of every layer in pinned host memory"),
    "decode_loop_b16_t128k_budget96": Workload(
        "decode_loop_b16_t128k_budget96", B=16, T=131072, Hq=32, G=8, k=63, n_init=1, n_local=32,
        layers=4, min_len=65536, windows=1, seed=1006,
        note="the real models' decode configuration: 96 blocks (1 initial, 32 local = 2048 "
             "tokens, 63 top-k) chosen on the 32/16 window grid, sequences of mixed lengths "
             "between 64K and 128K tokens"),
    "prefill_b4_t128k_c2k": Workload(
        "prefill_b4_t128k_c2k", B=4, T=131072, Hq=32, G=8, k=64, nq=2048, seed=1004,
        note="prefill chunk of 2048 tokens at the end of a 128K sequence"),
}

# selection-only sweep: compressed-key block counts x batch sizes, 8 groups
SWEEP_NB = (128, 256, 512, 1024, 2048, 4096, 8192, 16384)
SWEEP_B = (1, 2, 4, 8, 16)
SWEEP_SEED = 1005


def decode_lengths(w: Workload) -> np.ndarray:
    """Tokens held by each sequence of a decode batch, int32 [B]: all T, or
    (min_len > 0) uniform integers in [min_len, T], seeded."""
    if w.min_len <= 0:
        return np.full(w.B, w.T, np.int32)
    return rng_for(w.seed, 2).integers(w.min_len, w.T + 1, size=w.B).astype(np.int32)


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields changed (smaller parity cases)."""
    return replace(w, **kw)


# --------------------------------------------------------------------------
# drawing
# --------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 raw bits, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rng_for(seed: int, stream: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, stream]))


def normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def plant_hot_blocks(K_f32: np.ndarray, F_bits: np.ndarray, w: Workload, rng) -> np.ndarray:
    """Shift every key row of ``w.planted`` random candidate blocks per (b, g)
    by 0.5 * F_g / |F_g| (F_g being the group's Forecast vector).

    K_f32: [B][G][T][d] float32 (modified in place); F_bits: [B][G][d] bf16 bits.
    Returns the planted block ids, int32 [B][G][planted].
    """
    B, G, T, d = K_f32.shape
    c_last = (T - 1) // w.blk
    lo, hi = w.n_init, c_last - w.n_local + 1          # candidate blocks of the last token
    Ff = bf16_bits_to_f32(F_bits).astype(np.float64)
    hot = np.empty((B, G, w.planted), np.int32)
    for b in range(B):
        for g in range(G):
            blocks = np.sort(rng.choice(np.arange(lo, hi), size=w.planted, replace=False))
            hot[b, g] = blocks
            direction = (0.5 * Ff[b, g] / np.linalg.norm(Ff[b, g])).astype(np.float32)
            for j in blocks:
                K_f32[b, g, j * w.blk:(j + 1) * w.blk, :] += direction
    return hot


def decode_inputs(w: Workload) -> dict:
    """One decode step of one layer: Q [B][Hq][d], F [B][G][d], K/V [B][G][T][d]."""
    rng = rng_for(w.seed)
    Q = normal_bf16(rng, (w.B, w.Hq, w.d))
    F = normal_bf16(rng, (w.B, w.G, w.d))
    K32 = rng.standard_normal((w.B, w.G, w.T, w.d), dtype=np.float32)
    hot = None
    if w.planted:
        hot = plant_hot_blocks(K32, F, w, rng_for(w.seed, 1))
    K = f32_to_bf16_bits(K32)
    del K32
    V = normal_bf16(rng, (w.B, w.G, w.T, w.d))
    out = dict(Q=Q, F=F, K=K, V=V)
    if hot is not None:
        out["hot"] = hot
    return out


def prefill_inputs(w: Workload) -> dict:
    """One prefill chunk: Q [B][nq][Hq][d], F [B][nq][G][d], K/V [B][G][T][d]."""
    rng = rng_for(w.seed)
    Q = normal_bf16(rng, (w.B, w.nq, w.Hq, w.d))
    F = normal_bf16(rng, (w.B, w.nq, w.G, w.d))
    K = normal_bf16(rng, (w.B, w.G, w.T, w.d))
    V = normal_bf16(rng, (w.B, w.G, w.T, w.d))
    return dict(Q=Q, F=F, K=K, V=V)


def sweep_inputs(NB: int, B: int, G: int = 8, Hq: int = 32, d: int = 128) -> dict:
    """Selection sweep point: Kc bf16 [B][G][NB][d] given directly, one Forecast
    vector per group F [B][G][d], and the group's query heads Q [B][Hq][d]."""
    rng = rng_for(SWEEP_SEED, NB * 64 + B)
    kc = normal_bf16(rng, (B, G, NB, d))
    F = normal_bf16(rng, (B, G, d))
    Q = normal_bf16(rng, (B, Hq, d))
    return dict(kc=kc, F=F, Q=Q)


def decode_loop_small_inputs(w: Workload) -> dict:
    """The decode loop at a size numpy can draw: per layer l, Q_l [B][Hq][d],
    F_l [B][G][d] (F_l selects layer l+1's blocks; F_{-1} selects layer 0's),
    and the layer's KV in the host layout [B][G][NB][2][blk][d]."""
    rng = rng_for(w.seed)
    L = w.layers
    Q = normal_bf16(rng, (L, w.B, w.Hq, w.d))
    F = normal_bf16(rng, (L + 1, w.B, w.G, w.d))          # F[0] is F_{-1}
    KV = normal_bf16(rng, (L, w.B, w.G, w.NB, 2, w.blk, w.d))
    return dict(Q=Q, F=F, KV=KV)


def torch_normal_bf16_(t, seed: int, chunk_elems: int = 1 << 28):
    """Fill a bf16 torch tensor (any device) with N(0,1) from torch's seeded
    generator on that device, chunk by chunk (plumbing only)."""
    import torch
    gen = torch.Generator(device=t.device)
    gen.manual_seed(seed)
    flat = t.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        flat[s:e].copy_(torch.randn(e - s, generator=gen, device=t.device, dtype=torch.float32))
    return t
