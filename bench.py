#!/usr/bin/env python
"""Benchmark of the SparDA decode hot path on B200.

Workload (one "step"): one decode token for B = 16 sequences at T = 131072
through a 4-layer loop, 32 query heads in 8 GQA groups, head_dim 128, blocks
of 64 tokens, top-k = 64 plus 1 initial and 2 local blocks.  Per layer l:
  select  -- the layer's Forecast vectors F_l score layer l+1's compressed
             keys (the last layer's select the next token's layer 0) and
             keep init U top-k U local;
  attend  -- the layer's queries attend over its selected 67 blocks.
Both need layer l-1 done and nothing from each other, so select(l) runs on a
side stream beside attention(l), and attention(l+1) waits for both.

value  : decode tokens/s with every input resident in HBM (K/V of all four
         layers, 34 GB, addressed by block id), timed with CUDA events.
e2e    : the same loop through the C ABI with the K/V cache in pinned host
         memory: per step Q and F are copied host->device, each layer's
         selected blocks are gathered over the host link into device slots
         on a side stream while the previous layer attends, and the output
         is copied device->host.  Cold sets: every step refetches.
"""
from __future__ import annotations

import argparse
import json
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_long_sparda_b200 import workloads as W  # noqa: E402

WORKLOAD = W.WORKLOADS["decode_loop_b16_t128k"]
METRIC = "decode tokens/s at B=16,T=128K (sparse attn+select, % HBM roofline); select us/layer"
GRAPH_STEPS = 5  # decode steps per CUDA graph replay in the timed region


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sparda", choices=["sparda", "reference"])
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-offload e2e leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="leave the prefill-chunk and selection-sweep summaries out of the line")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="bound on the oracle's CPU-baseline sample")
    ap.add_argument("--prefill", action="store_true",
                    help="also measure the prefill chunk workload (B=4, T=128K, 2048 query "
                         "tokens): compress, per-token select and sparse attention; prints "
                         "an extra JSON line")
    ap.add_argument("--sweep", action="store_true",
                    help="also measure the selection-only sweep (Kc blocks 128..16384 x "
                         "batch 1..16, Forecast vs the 4-head baseline selector); prints an "
                         "extra JSON line")
    ap.add_argument("--windows", action="store_true",
                    help="also measure the window grid of the real models (32-token windows "
                         "at stride 16, max-pooled to blocks): window compression, decode "
                         "selection at B=16, T=128K, and the prefill chunk's selection; prints "
                         "an extra JSON line")
    ap.add_argument("--real-model", action="store_true",
                    help="also measure the real models' decode configuration: 96-block sets "
                         "(1 initial, 32 local, 63 top-k) on the window grid, 16 sequences of "
                         "mixed lengths (64K..128K), 4 layers; prints an extra JSON line")
    ap.add_argument("--head-softmax", action="store_true",
                    help="also measure the original selector in its per-head softmax form "
                         "(each of a group's 4 query heads softmax-normalised over the seen "
                         "keys, summed) at B=16, T=128K on block keys and on window keys, "
                         "beside Forecast and the summed-score baseline on the same keys; "
                         "prints an extra JSON line")
    ap.add_argument("--only", choices=["prefill", "sweep", "windows", "real-model", "head-softmax"],
                    help="run this one leg alone (no decode loop) and print its JSON line")
    ap.add_argument("--profile-case", action="store_true",
                    help="run three passes of one decode layer (select, then attention) at "
                         "B=8 with the bench's other shapes (4.3 GB of K/V, 140 MB of selected "
                         "K/V per attention launch), then two passes of a 512-token prefill "
                         "chunk of one sequence, then two cold host gathers of one layer at B=2 "
                         "(1.1 GB pinned) and two cached selections (cold, then warm), then two head-softmax selections each on one "
                         "layer of block keys and of window keys at B=16, T=128K, and exit: "
                         "the small cases ncu captures")
    return ap.parse_args()


# --------------------------------------------------------------------------
# process plumbing
# --------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, local):
    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))


def _on_gpu():
    import torch
    return torch.cuda.is_available()


def max_over_ranks(x: float, world: int) -> float:
    """The largest value of x over all ranks (timings: the slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    import torch
    if _on_gpu():
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if _on_gpu():
        torch.cuda.synchronize()


def replica_value(tokens_per_replica: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job decode throughput of `world` independent replicas: every
    replica decodes its own batch, so the job's tokens per step are the sum
    over replicas, and the step takes as long as the slowest replica."""
    return tokens_per_replica * world / (ms_per_step_max / 1e3)


class ClockSampler:
    """nvidia-smi clock/throttle samples taken while the timed region runs."""

    def __init__(self, index: int):
        self.path = tempfile.mktemp(prefix="sparda_clocks_", suffix=".csv")
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            cmd = ["nvidia-smi", "-i", str(index), "--query-gpu=" + q,
                   "--format=csv,noheader,nounits", "-lms", "50"]
            if shutil.which("stdbuf"):
                cmd = ["stdbuf", "-oL"] + cmd        # line-buffered, so nothing is lost at stop
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        with open(self.path) as f:
            out = summarize_clock_samples(f)
        os.unlink(self.path)
        return out


def summarize_clock_samples(lines) -> dict:
    """nvidia-smi CSV rows (index, clocks.sm, clocks.max.sm, power.draw, the
    active-reasons mask, then hw_slowdown, hw_thermal_slowdown,
    sw_thermal_slowdown, sw_power_cap as "Active" / "Not Active") -> the
    median SM clock, the max clock and every reason seen active."""
    sm, smax, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in lines:
        c = [x.strip() for x in line.split(",")]
        if len(c) < 9:
            continue
        try:
            sm.append(float(c[1]))
            smax = float(c[2])
        except ValueError:
            continue
        for n, v in zip(names, c[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
            "reasons": sorted(reasons), "samples": len(sm)}


def measured_peaks(path=None):
    """The measured HBM copy bandwidth (GB/s) the driver wrote, else the
    earlier pool measurement, with which of the two it is."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def measured_bf16_peaks(path=None):
    """(burst, sustained) dense bf16 TFLOP/s: the driver's measurement, else
    the earlier pool measurement, with which of the two it is."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback"


# --------------------------------------------------------------------------
# the decode loop on one GPU
# --------------------------------------------------------------------------

class DecodeLoop:
    def __init__(self, w: W.Workload, with_host: bool, seed_offset: int = 0):
        import torch
        from block_sparse_long_sparda_b200 import abi
        self.torch, self.abi, self.w = torch, abi, w
        dev = torch.device("cuda")
        B, G, Hq, d, L, NB, S = w.B, w.G, w.Hq, w.d, w.layers, w.NB, w.S
        # per-sequence lengths (a length mix), else every sequence holds T tokens
        self.lens = W.decode_lengths(w)
        self.seq_len = None
        if w.min_len > 0:
            self.seq_len = torch.from_numpy(self.lens).to(dev)
        self.p = abi.make_params(B, Hq, G, w.T, w.k, w.n_init, w.n_local, seq_len=self.seq_len)
        seed = w.seed + 1000 * seed_offset
        self.blk_elems = 2 * w.blk * d                      # one K|V block pair
        # K/V cache of every layer, host layout [L][B][G][NB][2][64][128]
        self.kv = torch.empty(L, B, G, NB, 2, w.blk, d, dtype=torch.bfloat16, device=dev)
        for l in range(L):
            W.torch_normal_bf16_(self.kv[l], seed * 16 + l)
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed * 16 + 15)
        self.Q = torch.randn(L, B, Hq, d, generator=gen, device=dev).to(torch.bfloat16)
        self.F = torch.randn(L, B, G, d, generator=gen, device=dev).to(torch.bfloat16)
        if w.windows:
            # window-grid keys of every layer (32-token windows at stride 16); the
            # interleaved K|V blocks give no constant row stride across a block
            # boundary, so the keys are drawn like the K/V they summarise
            self.kc = None
            self.NW = (w.T - 32) // 16 + 1
            self.kw = torch.empty(L, B, G, self.NW, d, dtype=torch.bfloat16, device=dev)
            for l in range(L):
                W.torch_normal_bf16_(self.kw[l], seed * 16 + 8 + l)
        else:
            # compressed keys of every layer (each block pooled as its own 64-token run)
            self.kc = torch.empty(L, B, G, NB, d, dtype=torch.bfloat16, device=dev)
            pc = abi.make_params(1, B * G * NB, B * G * NB, w.blk, 1)
            for l in range(L):
                abi.sparda_compress_keys(pc, self.kv[l], self.blk_elems, d, None, self.kc[l])
        self.idx = torch.empty(L, B, G, S, dtype=torch.int32, device=dev)
        self.O = torch.empty(L, B, Hq, d, dtype=torch.bfloat16, device=dev)
        op = abi.SPARDA_OP_SELECT_WINDOWS if w.windows else abi.SPARDA_OP_SELECT
        self.ws_sel = [abi.workspace(op, self.p, 1, 1) for _ in range(L)]
        self.ws_att = abi.workspace(abi.SPARDA_OP_ATTN_DECODE, self.p)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        # layer 0's set comes from the previous token's last layer
        self.select(L - 1)
        self.compute = torch.cuda.current_stream()
        # resident step: attention on a high-priority stream, selection beside it
        self.main = torch.cuda.Stream(priority=-1)
        self.side_sel = torch.cuda.Stream(priority=0)
        self.ev_pre = [torch.cuda.Event() for _ in range(L)]
        self.ev_sel = [torch.cuda.Event() for _ in range(L)]
        self.host_kv = None
        self.cached_sel_first = False  # the cached step's selection stream (setup_cache)
        if with_host:
            self._setup_host()
        torch.cuda.synchronize()

    # ---- resident: all K/V in HBM, addressed by block id ----
    def select(self, l):
        """Layer l's Forecast vector picks layer l+1's blocks."""
        w, nxt = self.w, (l + 1) % self.w.layers
        if w.windows:
            self.abi.sparda_forecast_select_windows(self.p, self.F[l], 1, 1, w.T - 1, self.kw[nxt],
                                                    32, 16, self.idx[nxt], self.ws_sel[l],
                                                    self.status)
        else:
            self.abi.sparda_forecast_select(self.p, self.F[l], 1, 1, w.T - 1, self.kc[nxt],
                                            self.idx[nxt], self.ws_sel[l], self.status)

    def attention(self, l):
        w = self.w
        kv = self.kv[l]
        self.abi.sparda_sparse_attn_decode(self.p, self.Q[l], kv, kv.view(-1)[w.blk * w.d:],
                                           w.NB * self.blk_elems, self.blk_elems, self.idx[l],
                                           self.abi.SPARDA_ADDR_LOGICAL, self.O[l], self.ws_att,
                                           self.status)

    def step_resident(self, before_layer=None):
        """One decode token through the L layers.  select(l) -- layer l's
        Forecast vectors picking layer l+1's blocks -- and attention(l) both
        need layer l-1 finished and nothing from each other, so select(l)
        runs on a side stream beside attention(l); attention(l+1) waits for
        both (the order of Algorithm 2, which picks the next layer's blocks
        before the current layer attends).  before_layer(l), when given, is
        launched on the main stream ahead of attention(l): the decode append
        of layer l's new K/V rows and keys.  select(l) does not wait for it,
        since it reads layer l+1's keys, which that append does not touch.
        Launch on ``self.main``."""
        torch = self.torch
        for l in range(self.w.layers):
            self.ev_pre[l].record(self.main)
            if before_layer is not None:  # on the main stream, ahead of attention(l)
                with torch.cuda.stream(self.main):
                    before_layer(l)
            self.side_sel.wait_event(self.ev_pre[l])
            with torch.cuda.stream(self.side_sel):
                self.select(l)
                self.ev_sel[l].record(self.side_sel)
            with torch.cuda.stream(self.main):
                self.attention(l)
            self.main.wait_event(self.ev_sel[l])

    # ---- host offload: K/V in pinned host memory, gathered into slots ----
    def _setup_host(self):
        torch, w = self.torch, self.w
        L = w.layers
        nbytes = self.kv.numel() * 2
        self.host_kv = torch.empty(self.kv.shape, dtype=torch.bfloat16)
        rc = torch.cuda.cudart().cudaHostRegister(self.host_kv.data_ptr(), nbytes, 0)
        if int(rc) != 0:
            raise RuntimeError("cudaHostRegister of %.1f GB failed (%s)" % (nbytes / 1e9, rc))
        self.host_kv.copy_(self.kv)
        dev = torch.device("cuda")
        self.slots = torch.empty(L, w.B, w.G, w.S, 2, w.blk, w.d, dtype=torch.bfloat16, device=dev)
        # initial and local blocks stay resident in their slots (the same every step
        # at a fixed decode position); top-k slots are refetched every step
        c = (w.T - 1) // w.blk
        for l in range(L):
            self.slots[l, :, :, 0] = self.kv[l, :, :, 0]
            for s in range(w.n_local):
                self.slots[l, :, :, w.S - w.n_local + s] = self.kv[l, :, :, c - w.n_local + 1 + s]
        self.side = torch.cuda.Stream()
        self.sel_ev = [torch.cuda.Event() for _ in range(L)]
        self.fetch_ev = [torch.cuda.Event() for _ in range(L)]
        self.h_Q = self.Q.cpu().pin_memory()
        self.h_F = self.F.cpu().pin_memory()
        self.h_O = torch.empty(self.O.shape, dtype=torch.bfloat16).pin_memory()
        # prime: layer 0's blocks for the first step
        self.abi.sparda_prefetch_blocks(self.p, self.host_kv[0], self.idx[0], self.slots[0], True, 0,
                                        self.status)
        for l in range(L):
            self.fetch_ev[l].record()

    def unregister(self):
        if self.host_kv is not None:
            self.torch.cuda.cudart().cudaHostUnregister(self.host_kv.data_ptr())
            self.host_kv = None

    def step_e2e(self):
        torch, abi, w = self.torch, self.abi, self.w
        L = w.layers
        self.Q.copy_(self.h_Q, non_blocking=True)
        self.F.copy_(self.h_F, non_blocking=True)
        bg = w.S * self.blk_elems
        for l in range(L):
            nxt = (l + 1) % L
            abi.sparda_forecast_select(self.p, self.F[l], 1, 1, w.T - 1, self.kc[nxt],
                                       self.idx[nxt], self.ws_sel[l], self.status)
            self.sel_ev[l].record(self.compute)
            self.side.wait_event(self.sel_ev[l])
            abi.sparda_prefetch_blocks(self.p, self.host_kv[nxt], self.idx[nxt], self.slots[nxt],
                                       True, 0, self.status, stream=self.side)
            self.fetch_ev[nxt].record(self.side)
            self.compute.wait_event(self.fetch_ev[l])
            sl = self.slots[l]
            abi.sparda_sparse_attn_decode(self.p, self.Q[l], sl, sl.view(-1)[w.blk * w.d:], bg,
                                          self.blk_elems, self.idx[l], abi.SPARDA_ADDR_SLOT,
                                          self.O[l], self.ws_att, self.status)
        self.h_O.copy_(self.O, non_blocking=True)

    # ---- host offload with a device slot cache: fetch only new blocks ----
    def setup_cache(self, C: int, sigma: float, n_steps: int, seed: int = 7):
        """C slots per (layer, b, g); the Forecast vectors of step t+1 are
        those of step t plus sigma * N(0, 1) noise, so consecutive steps
        select mostly the same blocks (a drift model of consecutive tokens;
        sigma = 0 keeps the sets fixed).  Each step's inputs -- the queries
        and Forecast vectors of every layer -- sit packed in pinned host
        memory, one buffer per step, and cross the link as one copy."""
        torch, w = self.torch, self.w
        L, dev = w.layers, torch.device("cuda")
        self.C = C
        self.cache = torch.empty(L, w.B, w.G, C, 2, w.blk, w.d, dtype=torch.bfloat16, device=dev)
        self.block_of = torch.full((L, w.B, w.G, C), -1, dtype=torch.int32, device=dev)
        self.hand = torch.zeros(L, w.B, w.G, dtype=torch.int32, device=dev)
        self.phys = torch.empty(L, w.B, w.G, w.S, dtype=torch.int32, device=dev)
        self.fetch = torch.zeros(L, w.B, w.G, w.S, dtype=torch.int32, device=dev)
        gen = torch.Generator()
        gen.manual_seed(seed)
        F = self.F.float().cpu()
        q = self.Q.cpu().reshape(-1)
        self.n_q = q.numel()
        steps = []
        for _ in range(n_steps):
            steps.append(torch.cat([q, F.to(torch.bfloat16).reshape(-1)]))
            F = F + sigma * torch.randn(F.shape, generator=gen)
        self.h_in = torch.stack(steps).pin_memory()          # [step][Q | F]
        self.d_in = torch.empty(2, self.h_in.shape[1], dtype=torch.bfloat16, device=dev)
        self.d_out = torch.empty((2,) + tuple(self.O.shape), dtype=torch.bfloat16, device=dev)
        self.h_out = torch.empty(self.O.shape, dtype=torch.bfloat16).pin_memory()
        self.copy = torch.cuda.Stream()
        # the stream of the fused selection, plan and fetch: beside the
        # attention at a lower priority (as in the resident step), or ahead
        # of it at a higher one, so the fetch of the misses starts early
        self.sel_cached = torch.cuda.Stream(priority=-1 if self.cached_sel_first else 0)
        self.ev_begin, self.ev_o = torch.cuda.Event(), torch.cuda.Event()
        self.ev_in = [torch.cuda.Event() for _ in range(2)]
        self.ev_dl = [torch.cuda.Event() for _ in range(2)]
        self._recorded = set()

    def step_inputs(self, t: int):
        """(Q, F, O) of step t: views of the step's device buffers."""
        w, b = self.w, t % 2
        Q = self.d_in[b, :self.n_q].view(self.Q.shape)
        F = self.d_in[b, self.n_q:].view(self.F.shape)
        return Q, F, self.d_out[b]

    def begin_cached(self, t: int):
        """Before a run of cached steps from step t: upload step t's inputs
        (each step uploads the next step's)."""
        self.d_in[t % 2].copy_(self.h_in[t % self.h_in.shape[0]])
        self.torch.cuda.synchronize()
        self._recorded = set()

    def end_cached(self, t_next: int):
        """After a run of cached steps: join the copies still in flight (the
        next step's inputs, the last step's outputs)."""
        main = self.torch.cuda.current_stream()
        for ev in (("in", t_next % 2), ("dl", (t_next - 1) % 2)):
            if ev in self._recorded:
                main.wait_event((self.ev_in if ev[0] == "in" else self.ev_dl)[ev[1]])
        self._recorded = set()

    def step_e2e_cached(self, t: int):
        """One decode step through the C ABI with the K/V cache in pinned host
        memory and a device slot cache.  Per layer, one launch selects the
        next layer's blocks, plans them against that layer's slots and
        copies only the misses from the host, on a side stream, while this
        layer attends from its slots.  Step t's inputs were
        uploaded during step t-1 (begin_cached for the first); this step
        uploads step t+1's into the other buffer and sends its outputs back
        while the next step runs.  The main stream never waits on the copy
        stream directly: the copies join the selection stream ahead of the
        last layer's selection, which the next step's first attention waits
        for.  Runs of steps are captured into one CUDA graph."""
        torch, abi, w = self.torch, self.abi, self.w
        L, C = w.layers, self.C
        main = torch.cuda.current_stream()
        cur, oth = t % 2, (t + 1) % 2
        # step t+1's inputs go into the other buffer, which step t-1 no longer reads
        self.ev_begin.record(main)
        self.copy.wait_event(self.ev_begin)
        with torch.cuda.stream(self.copy):
            self.d_in[oth].copy_(self.h_in[(t + 1) % self.h_in.shape[0]], non_blocking=True)
            self.ev_in[oth].record(self.copy)
        self._recorded.add(("in", oth))
        Q, F, O = self.step_inputs(t)
        for l in range(L):
            nxt = (l + 1) % L
            self.ev_pre[l].record(main)
            self.sel_cached.wait_event(self.ev_pre[l])
            if l == L - 1:
                # the copies step t+1 depends on -- its inputs, issued at this
                # step's start, and step t-1's outputs leaving the buffer step
                # t+1 writes -- join here, long after they ended; attention(0)
                # of step t+1 waits for this selection anyway.  The copy
                # stream runs in order and issued step t-1's outputs before
                # step t+1's inputs, so the inputs' event covers both
                if ("in", oth) in self._recorded:
                    self.sel_cached.wait_event(self.ev_in[oth])
                elif ("dl", oth) in self._recorded:
                    self.sel_cached.wait_event(self.ev_dl[oth])
            with torch.cuda.stream(self.sel_cached):
                abi.sparda_forecast_select_cached(self.p, F[l], 1, w.T - 1, self.kc[nxt],
                                                  self.idx[nxt], self.ws_sel[l], C,
                                                  self.block_of[nxt], self.hand[nxt],
                                                  self.phys[nxt], self.fetch[nxt],
                                                  self.host_kv[nxt], self.cache[nxt],
                                                  self.status)
                self.fetch_ev[nxt].record(self.sel_cached)
            if l > 0:  # layer 0's blocks were joined at the end of the previous step
                main.wait_event(self.fetch_ev[l])
            abi.sparda_sparse_attn_decode_cached(self.p, C, Q[l], self.cache[l], self.idx[l],
                                                 self.phys[l], O[l], self.ws_att, self.status)
        # the outputs go back while the next step runs
        self.ev_o.record(main)
        self.copy.wait_event(self.ev_o)
        with torch.cuda.stream(self.copy):
            self.h_out.copy_(O, non_blocking=True)
            self.ev_dl[cur].record(self.copy)
        self._recorded.add(("dl", cur))
        main.wait_event(self.fetch_ev[0])

    def cached_steps(self, t0: int, n: int):
        """Steps t0 .. t0+n-1 back to back (one graph when captured)."""
        for t in range(t0, t0 + n):
            self.step_e2e_cached(t)
        self.end_cached(t0 + n)

    def prime_cache(self):
        """Cold start: plan and fetch layer 0's current set."""
        w = self.w
        self.abi.sparda_cache_plan(self.p, self.C, self.idx[0], self.block_of[0], self.hand[0],
                                   self.phys[0], self.fetch[0], self.status)
        self.abi.sparda_prefetch_cached(self.p, self.C, self.host_kv[0], self.idx[0], self.phys[0],
                                        self.fetch[0], self.cache[0], 0, self.status)
        self.torch.cuda.synchronize()

    # algorithmic bytes per launch
    def _ncand(self):
        """Candidate blocks of each sequence's query (its last token)."""
        w = self.w
        c = (self.lens.astype(np.int64) - 1) // w.blk
        return np.maximum(0, c - w.n_local + 1 - w.n_init)

    def bytes_select(self):
        """Key rows the selection must read: one per candidate block, or on the
        window grid the three windows inside each candidate block."""
        w = self.w
        rows = self._ncand() * (3 if w.windows else 1)
        return int(w.G * (rows.sum() * w.d * 2 + w.B * (w.d * 2 + w.S * 4)))

    def bytes_attn(self):
        """The K|V blocks of every set (full sets: each sequence has more
        candidates than k), plus Q, O and the lists."""
        w = self.w
        n_sel = np.minimum(self._ncand(), w.k) + w.n_init + w.n_local
        return int(w.G * n_sel.sum() * self.blk_elems * 2 + 2 * w.B * w.Hq * w.d * 2
                   + w.B * w.G * w.S * 4)


PROFILE_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles")
KERNEL_SOURCES = {
    "attn_tc_kernel": ["attn_decode.cu", "tc.cuh", "common.cuh"],
}


def kernel_source_hash(kernel):
    """Hash of the kernel's sources with comments and blank space removed, so
    that an edit of comments alone does not retire a profile."""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "block_sparse_long_sparda_b200",
                        "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, algorithmic_bytes):
    """DRAM bytes (read + write) per full launch from the committed ncu
    summary of this kernel, or None when there is none or the kernel's
    sources changed since it was taken."""
    import re
    for name in sorted(os.listdir(PROFILE_DIR)) if os.path.isdir(PROFILE_DIR) else []:
        if not name.startswith(kernel):
            continue
        with open(os.path.join(PROFILE_DIR, name)) as f:
            text = f.read()
        m_hash = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]{16})", text)
        m_tr = re.search(r"dram_bytes_per_full_launch:\s*([0-9]+)", text)
        if m_hash and m_tr and m_hash.group(1) == kernel_source_hash(kernel):
            return int(m_tr.group(1))
    return None


def time_steps(fn, steps, world):
    import torch
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        fn()
    end.record()
    end.synchronize()
    ms = start.elapsed_time(end)
    barrier(world)
    return max_over_ranks(ms, world)


# --------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands, on a bounded sample
# --------------------------------------------------------------------------

class OracleDecodeSample:
    """The decode loop's arithmetic on the fp64 oracle, for every sequence of
    the batch: per layer, the oracle's Forecast selection of the next layer's
    blocks for all B x G (sequence, group) problems, and its sparse attention
    of all B x Hq heads over the layer's current sets.  Inputs are given as
    host arrays: the compressed keys of every layer [L][B][G][NB][d], the
    Forecast vectors [L][B][G][d], the queries [L][B][Hq][d], and the K|V
    blocks of each layer's sets gathered in list order [L][B][G][S][2][blk][d]
    (the attention addresses entry s at position s; every key of a decode set
    precedes the query, so the causal mask never applies and the result is
    the attention over the blocks themselves)."""

    def __init__(self, w, kc, F, Q, kv_sets, idx0):
        self.w, self.kc, self.F, self.Q, self.kv, self.idx0 = w, kc, F, Q, kv_sets, idx0
        self.slot_idx = np.broadcast_to(np.arange(w.S, dtype=np.int32),
                                        (w.B, 1, w.G, w.S)).copy()

    def step(self):
        import oracle
        w = self.w
        L, B, G, d, blk, S = w.layers, w.B, w.G, w.d, w.blk, w.S
        for l in range(L):
            nxt = (l + 1) % L
            oracle.select(self.F[l].reshape(B, 1, G, 1, d), self.kc[nxt], w.k, w.n_init,
                          w.n_local, w.T - 1, blk)
            flat = self.kv[l].reshape(-1)
            oracle.sparse_attention(self.Q[l].reshape(B, 1, w.Hq, d), flat, flat[blk * d:],
                                    self.slot_idx, w.T - 1, w.T, blk,
                                    bg_stride=S * 2 * blk * d, blk_stride=2 * blk * d, G=G)

    def time(self, seconds: float, threads: int | None = None, max_reps: int = 1000,
             min_reps: int = 1):
        """(steps per second, reps, seconds) of back-to-back steps; threads
        bounds the oracle's thread pool (None: every host core)."""
        old = os.environ.get("SPARDA_ORACLE_THREADS")
        if threads is not None:
            os.environ["SPARDA_ORACLE_THREADS"] = str(threads)
        try:
            reps, t0 = 0, time.perf_counter()
            while True:
                self.step()
                reps += 1
                el = time.perf_counter() - t0
                if (el >= seconds and reps >= min_reps) or reps >= max_reps:
                    break
        finally:
            if threads is not None:
                if old is None:
                    os.environ.pop("SPARDA_ORACLE_THREADS", None)
                else:
                    os.environ["SPARDA_ORACLE_THREADS"] = old
        return reps / el, reps, el


def oracle_sets(w, kc, F):
    """Every layer's current sets, as the loop holds them at the start of a
    step: layer l's blocks were picked by layer l-1's Forecast vectors (layer
    0's by the last layer's).  [L][B][G][S]"""
    import oracle
    L, B, G, d = w.layers, w.B, w.G, w.d
    return np.stack([oracle.select(F[(l - 1) % L].reshape(B, 1, G, 1, d), kc[l], w.k, w.n_init,
                                   w.n_local, w.T - 1, w.blk)[0][:, 0] for l in range(L)])


def oracle_sample_from_loop(loop: DecodeLoop) -> OracleDecodeSample:
    """The oracle's inputs taken from the GPU loop's own buffers: the same
    compressed keys, Forecast vectors and queries, and the K|V blocks of the
    sets the oracle itself picks (gathered on the device, outside any timing)."""
    import torch
    w = loop.w

    def bits(t):
        return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    kc = [bits(loop.kc[l]) for l in range(w.layers)]
    F, Q = bits(loop.F), bits(loop.Q)
    sets = oracle_sets(w, kc, F)
    kv = []
    for l in range(w.layers):
        ids = torch.from_numpy(np.maximum(sets[l], 0).astype(np.int64)).to(loop.kv.device)
        flat = loop.kv[l].reshape(w.B * w.G, w.NB, -1)
        g = torch.gather(flat, 1, ids.reshape(w.B * w.G, w.S, 1).expand(-1, -1, flat.shape[2]))
        kv.append(bits(g).reshape(w.B, w.G, w.S, 2, w.blk, w.d))
    return OracleDecodeSample(w, kc, F, Q, kv, sets[0])


def oracle_sample_synthetic(w, seed: int) -> OracleDecodeSample:
    """The same sample with inputs drawn on the host (numpy, seeded): block
    keys N(0, 1/64) like the means of 64 N(0, 1) keys, Forecast vectors and
    queries N(0, 1), and N(0, 1) K|V for the blocks of each layer's sets."""
    import oracle  # noqa: F401  (the oracle is built on first use)
    L, B, G, d = w.layers, w.B, w.G, w.d
    rng = W.rng_for(seed, 99)
    kc = [W.f32_to_bf16_bits(rng.standard_normal((B, G, w.NB, d), dtype=np.float32) / 8)
          for _ in range(L)]
    F = W.normal_bf16(rng, (L, B, G, d))
    Q = W.normal_bf16(rng, (L, B, w.Hq, d))
    sets = oracle_sets(w, kc, F)
    kv = [W.normal_bf16(rng, (B, G, w.S, 2, w.blk, d)) for _ in range(L)]
    return OracleDecodeSample(w, kc, F, Q, kv, sets[0])


def oracle_baseline(loop: DecodeLoop, seconds: float):
    """The fp64 oracle as it stands, timed on the host cores on the whole
    batch of the GPU loop (all 16 sequences, 4 layers, the same inputs),
    with every host core and then with one."""
    import oracle
    smp = oracle_sample_from_loop(loop)
    w = loop.w
    rate, reps, el = smp.time(seconds, min_reps=2)
    rate1, reps1, el1 = smp.time(0.0, threads=1, max_reps=1)
    return {"value": w.B * rate, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "all %d sequences x %d layers per step (select of every (sequence, group) "
                      "over %d blocks + attention of every head over its %d-block set), %d steps, "
                      "%.1f s; inputs are the GPU loop's (K|V of the oracle's own sets)"
                      % (w.B, w.layers, w.NB, w.S, reps, el),
            "one_core": {"value": w.B * rate1, "unit": "tokens/s", "cores": 1,
                         "steps": reps1, "seconds": round(el1, 2)}}


# --------------------------------------------------------------------------
# arms
# --------------------------------------------------------------------------

def run_sparda(args):
    import torch
    from block_sparse_long_sparda_b200 import abi
    rank, world, local = dist_env()
    init_dist(world, local)
    from block_sparse_long_sparda_b200 import build
    build.build()
    w = WORKLOAD
    want_e2e = not args.no_e2e
    loop = DecodeLoop(w, with_host=False, seed_offset=rank)
    # the host-offload legs pin a 32 GiB host copy of this rank's K/V; every
    # rank runs them or none does (their timings meet at collectives)
    e2e_skip = None
    if want_e2e:
        try:
            loop._setup_host()
        except (RuntimeError, MemoryError) as exc:
            e2e_skip = "pinned host copy of the K/V unavailable on rank %d: %s" % (rank, exc)
            loop.unregister()
        if max_over_ranks(1.0 if e2e_skip else 0.0, world) > 0:
            want_e2e = False
            loop.unregister()
            e2e_skip = e2e_skip or "pinned host copy of the K/V unavailable on another rank"
    L = w.layers

    # every resident-step launch, its graph capture and its timing are on the
    # loop's high-priority main stream (selection forks onto a side stream)
    with torch.cuda.stream(loop.main):
        for _ in range(max(args.warmup, 3)):
            loop.step_resident()
        # the whole 4-layer step is replayed from a CUDA graph: no host work and
        # no launch gaps inside the timed region.  A graph of GRAPH_STEPS
        # consecutive steps (the step has no host dependency) pays one graph
        # launch per GRAPH_STEPS steps; single-step replays make up the rest.
        step, graph, graph_m = loop.step_resident, None, None
        try:
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=loop.main):
                loop.step_resident()
            graph.replay()
            graph_m = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_m, stream=loop.main):
                for _ in range(GRAPH_STEPS):
                    loop.step_resident()
            graph_m.replay()
            torch.cuda.synchronize()
            step = graph.replay
        except Exception as exc:  # keep eager launches, and say so in the line
            print("note: graph capture failed (%s); timing eager launches" % exc, file=sys.stderr)
            graph = graph_m = None
            torch.cuda.synchronize()

        def run_steps(n):
            """n steps: multi-step graph replays, then single steps."""
            if graph_m is not None:
                for _ in range(n // GRAPH_STEPS):
                    graph_m.replay()
                n %= GRAPH_STEPS
            for _ in range(n):
                step()
        for _ in range(max(args.warmup, 3)):
            step()
        # clocks are sampled over a ~1 s busy window that contains the timed steps
        # (untimed padding before and after keeps the GPU in the same state)
        est = time_steps(step, 5, world) / 5
        pad = max(1, int(400.0 / max(est, 1e-3)))
        clocks = ClockSampler(local)
        for _ in range(pad):
            step()
        ms = time_steps(lambda: run_steps(args.steps), 1, world)
        for _ in range(pad):
            step()
        torch.cuda.synchronize()
        clk = clocks.stop()
        # per-kernel durations: each kernel alone, back to back over the four
        # layers on the same stream (as launched in the step), CUDA events around
        # the whole run; events between kernels would break the programmatic
        # overlap of consecutive launches
        def kernel_loop(which):
            for l in range(L):
                if which == "select":
                    loop.select(l)
                else:
                    loop.attention(l)
        kern_us = {}
        for which in ("select", "attention"):
            for _ in range(3):
                kernel_loop(which)
            kms = time_steps(lambda: kernel_loop(which), args.steps, world)
            kern_us[which] = kms / (args.steps * L) * 1e3
        # decode append (new K/V rows + the incremental compressed key), timed
        # from a CUDA graph by writing every layer's last-token rows back
        # unchanged
        pos = w.T - 1
        c_last, r_last = pos // w.blk, pos % w.blk
        k_new = [loop.kv[l, :, :, c_last, 0, r_last].contiguous() for l in range(L)]  # [B][G][d]
        v_new = [loop.kv[l, :, :, c_last, 1, r_last].contiguous() for l in range(L)]

        def append_all():
            for l in range(L):
                kv = loop.kv[l]
                abi.sparda_append_kv(loop.p, pos, k_new[l], v_new[l], kv,
                                     kv.view(-1)[w.blk * w.d:], w.NB * loop.blk_elems,
                                     loop.blk_elems, None, loop.kc[l])
        for _ in range(3):
            append_all()
        torch.cuda.synchronize()
        g_app = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_app, stream=loop.main):
            append_all()
        kern_us["append"] = time_steps(g_app.replay, args.steps, world) / (args.steps * L) * 1e3
        del g_app
    st = int(loop.status.item())

    ms_step = ms / args.steps
    value = replica_value(w.B, world, ms_step)
    peak, peak_kind = measured_peaks()
    att_us = kern_us["attention"]
    sel_us = kern_us["select"]
    att_gbs = loop.bytes_attn() / (att_us * 1e-6) / 1e9
    sel_gbs = loop.bytes_select() / (sel_us * 1e-6) / 1e9
    layer_bytes = loop.bytes_attn() + loop.bytes_select()
    step_gbs = L * layer_bytes / (ms_step * 1e-3) / 1e9
    traffic = profiled_traffic("attn_tc_kernel", loop.bytes_attn())
    b_attn = loop.bytes_attn()

    e2e = {"unavailable": e2e_skip} if e2e_skip else None
    if want_e2e:
        for _ in range(max(args.warmup, 3)):
            loop.step_e2e()
        e_steps = max(3, min(args.steps, 10))
        e_ms = time_steps(loop.step_e2e, e_steps, world) / e_steps
        fetched = w.B * w.G * w.k * loop.blk_elems * 2 * L
        link_peak = host_link_peak_gbps()
        e2e = {"value": w.B * world / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(loop.Q.numel() * 2 + loop.F.numel() * 2),
               "d2h_bytes_per_step": int(loop.O.numel() * 2),
               "ms_per_step": e_ms,
               "host_link_bytes_per_step": fetched,
               "host_link_GBps": fetched / (e_ms * 1e-3) / 1e9,
               "host_link_peak_GBps": link_peak,
               "host_link_frac": fetched / (e_ms * 1e-3) / 1e9 / link_peak,
               # the wait the gather adds to each layer over the all-resident step
               "exposed_wait_us_per_layer": (e_ms - ms_step) * 1e3 / L,
               "note": "K/V in pinned host memory; every layer's top-k blocks gathered over the "
                       "host link on a side stream (cold sets, no reuse across steps)"}
        e2e["slot_cache"] = run_slot_cache_legs(loop, args, world, ms_step)
        loop.unregister()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(loop, args.cpu_seconds)
    del loop
    torch.cuda.empty_cache()
    # the prefill chunk and the selection sweep, summarised in the same line
    prefill = sweep = None
    if world == 1 and not args.no_extra:
        prefill = prefill_summary(run_prefill(args.steps, with_oracle=rank == 0))
        sweep = sweep_summary(with_oracle=rank == 0)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "layers": L, "Hq": w.Hq,
                       "G": w.G, "d": w.d, "block": w.blk, "k": w.k, "n_init": w.n_init,
                       "n_local": w.n_local, "parallelism": "replicas" if world > 1 else "single",
                       "kv": "all layers resident in HBM (34.4 GB), read by block id",
                       "streams": "select(l) on a side stream beside attention(l); "
                                  "attention(l+1) waits for both",
                       "l2": "inputs larger than L2: 281 MB of selected K/V per layer, 4 layers"},
            "select_us_per_layer": sel_us,
            "append_us_per_layer": kern_us["append"],
            "attn_us_per_layer": att_us,
            "select_GBps": sel_gbs,
            "step_GBps": step_gbs,
            "step_hbm_frac": step_gbs / peak,
            "roofline": {"bound": "hbm", "kernel": "attn_tc_kernel", "achieved": att_gbs,
                         "peak": peak, "unit": "GB/s", "frac": att_gbs / peak,
                         "traffic": traffic, "peak_kind": peak_kind,
                         "bytes_per_launch": b_attn},
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "prefill": prefill,
            "sweep": sweep,
            "gpu_launches": args.steps * L * 2,
            "cuda_graph": graph is not None,
            "graph_steps": GRAPH_STEPS if graph_m is not None else 1,
            "device_status": st,
        }
        print(json.dumps(line), flush=True)
    if rank == 0 and world == 1 and args.prefill:
        print(json.dumps(run_prefill(args.steps)), flush=True)
    if rank == 0 and world == 1 and args.sweep:
        print(json.dumps(run_sweep()), flush=True)
    if rank == 0 and world == 1 and args.windows:
        print(json.dumps(run_windows(args.steps)), flush=True)
    if rank == 0 and world == 1 and args.real_model:
        print(json.dumps(run_real_model(args.steps)), flush=True)
    if rank == 0 and world == 1 and args.head_softmax:
        print(json.dumps(run_head_softmax(args.steps)), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_slot_cache_legs(loop, args, world, resident_ms, sigmas=(0.0, 0.01, 0.03, 0.1)):
    """The e2e loop with a device slot cache (2S slots per layer and group)
    under a few drift rates of the Forecast vectors between decode steps:
    per-step time, the share of top-k blocks that still cross the host
    link, and the step time against the all-resident step.  Timed as one
    CUDA graph of the timed steps (each uploads the next step's inputs and
    sends its outputs back), after a warm-up graph of the steps before."""
    import torch
    w = loop.w
    L = w.layers
    out = []
    e_steps = max(3, min(args.steps, 10))
    warm = max(args.warmup, 3)
    for sigma in sigmas:
        n = warm + 2 * e_steps + 1
        loop.setup_cache(2 * w.S, sigma, n)
        # launched and captured like the resident step: attention on the
        # high-priority main stream, unless the selection goes first
        cap = torch.cuda.Stream() if loop.cached_sel_first else loop.main
        with torch.cuda.stream(cap):  # one eager step first: every launch's setup is done
            loop.prime_cache()
            loop.begin_cached(0)
            loop.cached_steps(0, 1)
        torch.cuda.synchronize()
        graphs = []
        with torch.cuda.stream(cap):
            for t0, cnt in ((0, warm), (warm, e_steps)):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cap):
                    loop.cached_steps(t0, cnt)
                graphs.append(g)
        torch.cuda.synchronize()
        loop.block_of.fill_(-1)   # capture enqueued nothing; start the cache cold again
        loop.hand.zero_()
        with torch.cuda.stream(cap):
            loop.prime_cache()
            loop.begin_cached(0)
            graphs[0].replay()
            ms = time_steps(graphs[1].replay, 1, world) / e_steps
            # the fetched share, on the steps that follow (run eagerly, untimed)
            fetched = 0
            t0 = warm + e_steps
            loop.begin_cached(t0)
            for t in range(t0, t0 + e_steps):
                loop.step_e2e_cached(t)
                torch.cuda.synchronize()
                fetched += int(loop.fetch.sum().item())
            loop.end_cached(t0 + e_steps)
        torch.cuda.synchronize()
        del graphs
        per_step = fetched / e_steps
        topk_entries = L * w.B * w.G * w.k
        out.append({"drift_sigma": sigma, "value": w.B * world / (ms / 1e3), "unit": "tokens/s",
                    "ms_per_step": ms, "fetched_blocks_per_step": per_step,
                    "fetched_frac_of_topk": per_step / topk_entries,
                    "host_link_bytes_per_step": int(per_step * loop.blk_elems * 2),
                    "h2d_bytes_per_step": int(loop.h_in.shape[1] * 2),
                    "d2h_bytes_per_step": int(loop.h_out.numel() * 2),
                    "step_vs_resident": ms / resident_ms,
                    "exposed_wait_us_per_layer": (ms - resident_ms) * 1e3 / L})
        del loop.cache, loop.block_of, loop.hand, loop.phys, loop.fetch, loop.h_in, loop.d_in
        del loop.d_out, loop.h_out
        torch.cuda.empty_cache()
    return out


def host_link_peak_gbps(nbytes=1 << 30, reps=5):
    """Pinned host -> device copy bandwidth (one large cudaMemcpyAsync, best
    of a few): the link peak the host gather is compared with."""
    import torch
    src = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dst = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    best = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dst.copy_(src, non_blocking=True)
        e1.record()
        e1.synchronize()
        best = max(best, nbytes / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del src, dst
    return best


def time_cold(fn, reps, warm=3):
    """Device time of one call with L2 flushed before it: a read of 256 MB
    (twice L2) runs before every call on the same stream.  A read leaves L2
    holding clean lines, so the timed call pays no write-back of the flush
    (a memset would leave ~126 MB of dirty lines behind).  CUDA events here
    tick in ~2 us steps, too coarse for a 10-30 us call, so `reps` (flush,
    call) pairs are timed as one span and `reps` flushes alone as another;
    the call's time is their difference over reps, the median of 3 trials."""
    import torch
    flush = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    sink = torch.zeros(reps, dtype=torch.float32, device="cuda")
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()

    def span(with_call):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(reps):
            torch.sum(flush, dim=0, out=sink[i])
            if with_call:
                fn()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) * 1e3
    span(True)
    span(False)
    trials = sorted((span(True) - span(False)) / reps for _ in range(3))
    del flush
    return trials[1]                               # us per call


def time_back_to_back(fn, steps, warm=3):
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    e1.synchronize()
    return e0.elapsed_time(e1) / steps * 1e3      # us per call


def time_graph(fn, steps, warm=3):
    """us per call of `steps` calls captured into one CUDA graph and replayed:
    for calls of a few tens of us, the host's per-call launch cost (tensor
    maps, argument marshalling) would otherwise set the pace."""
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(steps):
                fn()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    us = time_back_to_back(g.replay, 3, warm=0) / steps
    del g
    return us


class PrefillChunk:
    """Prefill chunk: B=4 sequences of T=131072 tokens whose last 2048 tokens
    are the queries (positions T-2048 .. T-1), one Forecast vector per token
    and group, K/V [B][G][T][128] in HBM."""

    def __init__(self, w: W.Workload = None):
        import torch
        from block_sparse_long_sparda_b200 import abi
        self.torch, self.abi = torch, abi
        w = w or W.WORKLOADS["prefill_b4_t128k_c2k"]
        self.w = w
        dev = torch.device("cuda")
        B, G, Hq, d, T, nq, NB, S = w.B, w.G, w.Hq, w.d, w.T, w.nq, w.NB, w.S
        self.p = abi.make_params(B, Hq, G, T, w.k, w.n_init, w.n_local)
        self.K = torch.empty(B, G, T, d, dtype=torch.bfloat16, device=dev)
        self.V = torch.empty(B, G, T, d, dtype=torch.bfloat16, device=dev)
        W.torch_normal_bf16_(self.K, w.seed * 16)
        W.torch_normal_bf16_(self.V, w.seed * 16 + 1)
        gen = torch.Generator(device=dev)
        gen.manual_seed(w.seed * 16 + 2)
        self.Q = torch.randn(B, nq, Hq, d, generator=gen, device=dev).to(torch.bfloat16)
        self.F = torch.randn(B, nq, G, d, generator=gen, device=dev).to(torch.bfloat16)
        self.kc = torch.empty(B, G, NB, d, dtype=torch.bfloat16, device=dev)
        self.idx = torch.empty(B, nq, G, S, dtype=torch.int32, device=dev)
        self.O = torch.empty(B, nq, Hq, d, dtype=torch.bfloat16, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws_sel = abi.workspace(abi.SPARDA_OP_SELECT, self.p, nq, 1)
        self.ws_att = abi.workspace(abi.SPARDA_OP_ATTN_PREFILL, self.p, nq, 1)
        self.q0 = T - nq

    def compress(self):
        w = self.w
        self.abi.sparda_compress_keys(self.p, self.K, w.T * w.d, w.d, None, self.kc)

    def select(self):
        self.abi.sparda_forecast_select(self.p, self.F, self.w.nq, 1, self.q0, self.kc, self.idx,
                                        self.ws_sel, self.status)

    def attention(self):
        w = self.w
        self.abi.sparda_sparse_attn_prefill(self.p, self.Q, w.nq, self.q0, self.K, self.V,
                                            w.T * w.d, w.d, self.idx, self.O, self.ws_att,
                                            self.status)

    def flops(self):
        """(select FLOPs, useful attention FLOPs) of one chunk."""
        w = self.w
        ncand = keys = 0
        for i in range(w.nq):
            pos = self.q0 + i
            nc = max(0, pos // w.blk - w.n_local + 1 - w.n_init)
            ncand += nc
            keys += (min(w.k, nc) + w.n_init + w.n_local - 1) * w.blk + pos % w.blk + 1
        return 2.0 * w.B * w.G * w.d * ncand, 4.0 * w.B * w.Hq * w.d * keys


def oracle_prefill_sample(pc, n_tok: int = 32):
    """The fp64 oracle on a bounded sample of the prefill chunk: the last
    n_tok query tokens of sequence 0, every group, per-token selection over
    the GPU's compressed keys and attention over the oracle's sets; the time
    is scaled to the whole chunk (B x nq tokens)."""
    import oracle
    import torch
    w = pc.w

    def bits(t):
        return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    K, V = bits(pc.K[:1]), bits(pc.V[:1])
    kc = bits(pc.kc[:1])
    F = bits(pc.F[:1, w.nq - n_tok:]).reshape(1, n_tok, w.G, 1, w.d)
    Q = bits(pc.Q[:1, w.nq - n_tok:])
    q0 = w.T - n_tok
    t0 = time.perf_counter()
    idx, _, _ = oracle.select(F, kc, w.k, w.n_init, w.n_local, q0, w.blk)
    t1 = time.perf_counter()
    oracle.sparse_attention(Q, K, V, idx, q0, w.T, w.blk)
    t2 = time.perf_counter()
    scale = w.B * w.nq / n_tok
    return {"select_us": (t1 - t0) * 1e6 * scale, "attn_us": (t2 - t1) * 1e6 * scale,
            "chunk_us": (t2 - t0) * 1e6 * scale, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "the last %d query tokens of sequence 0, all %d groups, timed once and "
                      "scaled by %d" % (n_tok, w.G, int(scale))}


def run_prefill(steps, with_oracle=False):
    pc = PrefillChunk()
    w = pc.w
    n = max(3, min(steps, 10))
    c_us = time_back_to_back(pc.compress, n)
    s_us = time_back_to_back(pc.select, n)
    a_us = time_back_to_back(pc.attention, n)
    st = int(pc.status.item())
    sel_flop, att_flop = pc.flops()
    cpu = oracle_prefill_sample(pc) if with_oracle else None
    return {
        "metric": "prefill chunk: compress, per-token Forecast select, sparse attention (us)",
        "workload": w.name, "B": w.B, "T": w.T, "nq": w.nq, "Hq": w.Hq, "G": w.G, "k": w.k,
        "compress_us": c_us, "compress_GBps": w.B * w.G * w.T * w.d * 2 / (c_us * 1e-6) / 1e9,
        "select_us": s_us, "select_TFLOPs": sel_flop / (s_us * 1e-6) / 1e12,
        "attn_us": a_us, "attn_useful_TFLOPs": att_flop / (a_us * 1e-6) / 1e12,
        "attn_gathered_GBps": w.B * w.nq * w.G * w.S * 2 * w.blk * w.d * 2 / (a_us * 1e-6) / 1e9,
        "chunk_us": s_us + a_us, "tokens_per_s": w.B * w.nq / ((s_us + a_us) * 1e-6),
        "device_status": st, "data": "synthetic", "dtype": "bf16", "cpu_baseline": cpu,
    }


def prefill_summary(r):
    """The prefill chunk's figures for the main JSON line."""
    burst, sustained, kind = measured_bf16_peaks()
    return {"workload": r["workload"], "select_us": round(r["select_us"], 1),
            "attn_us": round(r["attn_us"], 1), "chunk_us": round(r["chunk_us"], 1),
            "tokens_per_s": round(r["tokens_per_s"], 1),
            "attn_useful_TFLOPs": round(r["attn_useful_TFLOPs"], 2),
            "attn_frac_of_bf16_peak": round(r["attn_useful_TFLOPs"] / burst, 4),
            "select_TFLOPs": round(r["select_TFLOPs"], 2),
            "compress_us": round(r["compress_us"], 1), "compress_GBps": round(r["compress_GBps"], 1),
            "bf16_peak_TFLOPs": burst, "peak_kind": kind, "device_status": r["device_status"],
            "cpu_baseline": r.get("cpu_baseline")}


def sweep_summary(with_oracle=False):
    """The selection sweep's two cuts for the main JSON line: every block
    count at B = 16, and every batch at NB = 2048; Forecast next to the
    4-head baseline selector on the same keys, L2 flushed before each call.
    with_oracle: also the fp64 oracle's Forecast selection time at NB = 2048
    and 16384, B = 16, on the same keys (one call each)."""
    pts = [(NB, 16) for NB in W.SWEEP_NB] + [(2048, B) for B in W.SWEEP_B if B != 16]
    r = run_sweep(pts, oracle_pts=[(2048, 16), (16384, 16)] if with_oracle else ())
    return {"points": [[p["NB"], p["B"], p["forecast_us"], p["baseline_us"], p["forecast_GBps"]]
                       for p in r["points"]],
            "columns": ["NB", "B", "forecast_us", "baseline_us", "forecast_GBps"],
            "cpu_baseline": r.get("oracle"),
            "timing": r["timing"], "clocks": r["clocks"]}


def run_windows(steps):
    """The window grid: decode selection at the decode loop's shapes and the
    prefill chunk's, plus the window compression of the chunk's keys."""
    import torch
    from block_sparse_long_sparda_b200 import abi
    dev = torch.device("cuda")
    n = max(3, min(steps, 20))
    out = {"metric": "window-grid selection (32-token windows, stride 16, max-pooled to blocks)",
           "data": "synthetic", "dtype": "bf16"}
    # decode: B=16, T=128K, one Forecast vector per group
    w = WORKLOAD
    NW = (w.T - 32) // 16 + 1
    p = abi.make_params(w.B, w.Hq, w.G, w.T, w.k, w.n_init, w.n_local)
    kws = []
    for s_ in range(2):  # two layers' window keys (536 MB), alternated
        kw = torch.empty(w.B, w.G, NW, w.d, dtype=torch.bfloat16, device=dev)
        W.torch_normal_bf16_(kw, 3000 + s_)
        kws.append(kw)
    gen = torch.Generator(device=dev)
    gen.manual_seed(3100)
    F = torch.randn(w.B, w.G, w.d, generator=gen, device=dev).to(torch.bfloat16)
    idx = torch.empty(w.B, w.G, w.S, dtype=torch.int32, device=dev)
    ws = [abi.workspace(abi.SPARDA_OP_SELECT_WINDOWS, p, 1, 1) for _ in range(2)]
    t = [0]

    def sel():
        l = t[0] & 1
        abi.sparda_forecast_select_windows(p, F, 1, 1, w.T - 1, kws[l], 32, 16, idx, ws[l])
        t[0] += 1
    us = time_graph(sel, n)
    # the three windows inside each candidate block (the straddling fourth
    # window of a block is never scored, and never read)
    ncand = (w.T - 1) // w.blk - w.n_local + 1 - w.n_init
    nbytes = w.B * w.G * ncand * 3 * w.d * 2
    out.update({"decode_select_us": us, "decode_select_GBps": nbytes / (us * 1e-6) / 1e9,
                "decode_window_key_bytes": nbytes})
    del kws
    torch.cuda.empty_cache()
    # prefill chunk: window compression of its keys and per-token selection
    pc = PrefillChunk()
    pw = pc.w
    NWp = (pw.T - 32) // 16 + 1
    kwp = torch.empty(pw.B, pw.G, NWp, pw.d, dtype=torch.bfloat16, device=dev)
    wsp = abi.workspace(abi.SPARDA_OP_SELECT_WINDOWS, pc.p, pw.nq, 1)
    c_us = time_back_to_back(lambda: abi.sparda_compress_windows(
        pc.p, pc.K, pw.T * pw.d, pw.d, 32, 16, None, kwp), n)
    s_us = time_back_to_back(lambda: abi.sparda_forecast_select_windows(
        pc.p, pc.F, pw.nq, 1, pc.q0, kwp, 32, 16, pc.idx, wsp), max(3, min(n, 10)))
    out.update({"prefill_compress_windows_us": c_us,
                "prefill_compress_windows_GBps": pw.B * pw.G * pw.T * pw.d * 2 / (c_us * 1e-6) / 1e9,
                "prefill_select_us": s_us})
    return out


def run_real_model(steps):
    """The real models' decode configuration in the 4-layer loop: 96-block
    sets (1 initial, 32 local, 63 top-k) chosen on the window grid, for 16
    sequences of mixed lengths (64K..128K tokens), all K/V resident.  The
    step is the resident step of the headline loop (select(l) beside
    attention(l)), replayed from a CUDA graph."""
    import torch
    w = W.WORKLOADS["decode_loop_b16_t128k_budget96"]
    loop = DecodeLoop(w, with_host=False)
    L = w.layers
    n = max(5, min(steps, 50))
    # the full decode order of a layer puts the append first: the new token's
    # K/V rows and its block key (sparda_append_kv), and the window it
    # completes (sparda_append_windows), each sequence at its own last position
    d, blk = w.d, w.blk
    k_new = [torch.randn(w.B, w.G, d, device="cuda").to(torch.bfloat16) for _ in range(L)]
    v_new = [torch.randn(w.B, w.G, d, device="cuda").to(torch.bfloat16) for _ in range(L)]
    kc_blocks = torch.empty(w.B, w.G, w.NB, d, dtype=torch.bfloat16, device="cuda")

    def append(l):
        kv = loop.kv[l]
        loop.abi.sparda_append_kv(loop.p, w.T - 1, k_new[l], v_new[l], kv, kv.view(-1)[blk * d:],
                                  w.NB * loop.blk_elems, loop.blk_elems, None, kc_blocks)
        loop.abi.sparda_append_windows(loop.p, w.T - 1, kv, w.NB * loop.blk_elems, loop.blk_elems,
                                       32, 16, None, loop.kw[l])

    with torch.cuda.stream(loop.main):
        for _ in range(3):
            loop.step_resident()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=loop.main):
            loop.step_resident()
        step_us = time_back_to_back(graph.replay, n)
        g_full = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_full, stream=loop.main):
            loop.step_resident(before_layer=append)
        full_us = time_back_to_back(g_full.replay, n)
        del g_full
        kern = {}
        for which in ("select", "attention"):
            fn = (lambda: [loop.select(l) for l in range(L)]) if which == "select" else \
                 (lambda: [loop.attention(l) for l in range(L)])
            kern[which] = time_graph(fn, n) / L
        del graph
    torch.cuda.synchronize()
    st = int(loop.status.item())
    peak, peak_kind = measured_peaks()
    b_att, b_sel = loop.bytes_attn(), loop.bytes_select()
    step_gbs = L * (b_att + b_sel) / (step_us * 1e-6) / 1e9
    out = {
        "metric": "decode tokens/s, real-model budget (96 blocks: 1 initial + 32 local + 63 "
                  "top-k on the 32/16 window grid), mixed sequence lengths",
        "value": w.B / (step_us * 1e-6), "unit": "tokens/s", "data": "synthetic", "dtype": "bf16",
        "config": {"workload": w.name, "B": w.B, "T_max": w.T, "lengths": [int(x) for x in loop.lens],
                   "layers": L, "Hq": w.Hq, "G": w.G, "k": w.k, "n_init": w.n_init,
                   "n_local": w.n_local, "selection": "window grid, 32 tokens at stride 16",
                   "l2": "inputs larger than L2: %.0f MB of selected K/V per layer" % (b_att / 1e6)},
        "step_us": step_us, "step_GBps": step_gbs, "step_hbm_frac": step_gbs / peak,
        "step_with_append_us": full_us,
        "value_with_append": w.B / (full_us * 1e-6),
        "select_us_per_layer": kern["select"],
        "select_GBps": b_sel / (kern["select"] * 1e-6) / 1e9,
        "attn_us_per_layer": kern["attention"],
        "attn_GBps": b_att / (kern["attention"] * 1e-6) / 1e9,
        "attn_hbm_frac": b_att / (kern["attention"] * 1e-6) / 1e9 / peak,
        "bytes_per_layer": {"attention": b_att, "select": b_sel},
        "peak": peak, "peak_kind": peak_kind, "device_status": st,
    }
    del loop
    torch.cuda.empty_cache()
    return out


def run_sweep(pts=None, oracle_pts=()):
    """Selection-only sweep: Forecast (one vector per group) next to the
    baseline selector (the group's 4 query heads, scores summed) on the same
    compressed keys.  pts: (NB, B) points, default every combination."""
    import torch
    from block_sparse_long_sparda_b200 import abi
    dev = torch.device("cuda")
    G, Hq, d, k = 8, 32, 128, 64
    points, o_pts = [], []
    clocks = ClockSampler(torch.cuda.current_device())
    if pts is None:
        pts = [(NB, B) for NB in W.SWEEP_NB for B in W.SWEEP_B]
    for NB, B in pts:
        T = NB * 64
        p = abi.make_params(B, Hq, G, T, k)
        kc = torch.empty(B, G, NB, d, dtype=torch.bfloat16, device=dev)
        W.torch_normal_bf16_(kc, W.SWEEP_SEED * 1000 + NB + B)
        gen = torch.Generator(device=dev)
        gen.manual_seed(W.SWEEP_SEED + NB * 64 + B)
        F = torch.randn(B, G, d, generator=gen, device=dev).to(torch.bfloat16)
        Qh = torch.randn(B, Hq, d, generator=gen, device=dev).to(torch.bfloat16)
        idx = torch.empty(B, G, k + 3, dtype=torch.int32, device=dev)
        ws1 = abi.workspace(abi.SPARDA_OP_SELECT, p, 1, 1)
        ws4 = abi.workspace(abi.SPARDA_OP_SELECT, p, 1, Hq // G)
        f_us = time_cold(
            lambda: abi.sparda_forecast_select(p, F, 1, 1, T - 1, kc, idx, ws1), 15)
        b_us = time_cold(
            lambda: abi.sparda_forecast_select(p, Qh, 1, Hq // G, T - 1, kc, idx, ws4), 15)
        nbytes = B * G * NB * d * 2
        points.append({"NB": NB, "B": B, "forecast_us": round(f_us, 2),
                       "baseline_us": round(b_us, 2),
                       "forecast_GBps": round(nbytes / (f_us * 1e-6) / 1e9, 1)})
        if (NB, B) in oracle_pts:
            import oracle
            kcb = kc.cpu().view(torch.int16).numpy().view(np.uint16)
            Fb = F.cpu().view(torch.int16).numpy().view(np.uint16).reshape(B, 1, G, 1, d)
            t0 = time.perf_counter()
            oracle.select(Fb, kcb, k, 1, 2, T - 1)
            o_pts.append({"NB": NB, "B": B, "forecast_us": (time.perf_counter() - t0) * 1e6,
                          "cores": oracle.num_threads(), "kind": "oracle"})
        del kc
    return {"metric": "selection-only sweep: Forecast vs 4-head baseline selector (us per call)",
            "G": G, "k": k, "points": points, "data": "synthetic", "dtype": "bf16",
            "timing": "15 calls, each after a 256 MB read that flushes L2, timed as one span "
                      "less a span of the 15 reads alone; median of 3 trials",
            "oracle": o_pts or None, "clocks": clocks.stop()}


class HeadSoftmaxCase:
    """The original selector in its per-head softmax form at the decode
    loop's shapes (B=16, G=8 groups of 4 query heads, T=131072, k=64 with 1
    initial and 2 local blocks), on block keys or on the window grid.  Three
    layers' keys are alternated, so a call never finds its keys in L2
    (201 MB of block keys, 805 MB of window keys)."""

    def __init__(self, windows: bool, n_layers: int = 3, w: W.Workload = None):
        import math
        import torch
        from block_sparse_long_sparda_b200 import abi
        self.abi = abi
        w = w or WORKLOAD
        self.w, self.windows, self.L = w, windows, n_layers
        dev = torch.device("cuda")
        self.nf = w.Hq // w.G
        self.NR = (w.T - 32) // 16 + 1 if windows else w.NB
        self.p = abi.make_params(w.B, w.Hq, w.G, w.T, w.k, w.n_init, w.n_local)
        self.kc = []
        for l in range(n_layers):
            kc = torch.empty(w.B, w.G, self.NR, w.d, dtype=torch.bfloat16, device=dev)
            W.torch_normal_bf16_(kc, 5000 + 10 * l + int(windows))
            self.kc.append(kc)
        gen = torch.Generator(device=dev)
        gen.manual_seed(5100 + int(windows))
        self.Q = torch.randn(w.B, w.G, self.nf, w.d, generator=gen, device=dev).to(torch.bfloat16)
        self.F = torch.randn(w.B, w.G, 1, w.d, generator=gen, device=dev).to(torch.bfloat16)
        self.tau = math.sqrt(w.d)
        self.idx = torch.empty(w.B, w.G, w.S, dtype=torch.int32, device=dev)
        op_h = abi.SPARDA_OP_HEAD_SOFTMAX_WINDOWS if windows else abi.SPARDA_OP_HEAD_SOFTMAX
        op_s = abi.SPARDA_OP_SELECT_WINDOWS if windows else abi.SPARDA_OP_SELECT
        self.ws_h = abi.workspace(op_h, self.p, 1, self.nf)
        self.ws_f = abi.workspace(op_s, self.p, 1, 1)
        self.ws_s = abi.workspace(op_s, self.p, 1, self.nf)
        self.t = 0

    def _next(self):
        l = self.t % self.L
        self.t += 1
        return self.kc[l]

    def head_softmax(self, kc=None):
        kc = self._next() if kc is None else kc
        w, a = self.w, self.abi
        if self.windows:
            a.sparda_head_softmax_select_windows(self.p, self.Q, self.nf, w.T - 1, self.tau, kc,
                                                 32, 16, self.idx, self.ws_h)
        else:
            a.sparda_head_softmax_select(self.p, self.Q, self.nf, w.T - 1, self.tau, kc,
                                         self.idx, self.ws_h)

    def scores(self, vecs, nf, ws):
        kc = self._next()
        w, a = self.w, self.abi
        if self.windows:
            a.sparda_forecast_select_windows(self.p, vecs, 1, nf, w.T - 1, kc, 32, 16, self.idx, ws)
        else:
            a.sparda_forecast_select(self.p, vecs, 1, nf, w.T - 1, kc, self.idx, ws)

    def key_bytes(self):
        """Keys of every row a decode query at T-1 sees (the softmax reads
        them all)."""
        return self.w.B * self.w.G * self.NR * self.w.d * 2


def run_head_softmax(steps):
    """The original selector's per-head softmax form next to Forecast and the
    summed-score baseline, on the same keys."""
    import torch
    n = max(6, min(steps, 30))
    peak, peak_kind = measured_peaks()
    out = {"metric": "decode selection, the original selector's per-head softmax form vs "
                     "Forecast (us per call, one layer)",
           "data": "synthetic", "dtype": "bf16", "peak": peak, "peak_kind": peak_kind}
    clocks = ClockSampler(torch.cuda.current_device())
    for windows in (False, True):
        c = HeadSoftmaxCase(windows)
        h_us = time_graph(c.head_softmax, n)
        f_us = time_graph(lambda: c.scores(c.F, 1, c.ws_f), n)
        s_us = time_graph(lambda: c.scores(c.Q, c.nf, c.ws_s), n)
        nb = c.key_bytes()
        key = "windows" if windows else "blocks"
        out[key] = {"B": c.w.B, "T": c.w.T, "G": c.w.G, "heads_per_group": c.nf, "k": c.w.k,
                    "key_rows": c.NR, "key_bytes": nb,
                    "head_softmax_us": h_us, "head_softmax_GBps": nb / (h_us * 1e-6) / 1e9,
                    "head_softmax_hbm_frac": nb / (h_us * 1e-6) / 1e9 / peak,
                    "forecast_us": f_us, "summed_heads_us": s_us,
                    "l2": "3 layers' keys alternated (%.0f MB)" % (3 * nb / 1e6)}
        del c
        torch.cuda.empty_cache()
    out["clocks"] = clocks.stop()
    return out


def run_profile_case():
    """One decode layer at B=8, three passes: the small case for ncu."""
    import torch
    from block_sparse_long_sparda_b200 import abi
    w = W.scaled(WORKLOAD, B=8, layers=2)
    loop = DecodeLoop(w, with_host=False)
    bg = w.NB * loop.blk_elems
    kv = loop.kv[0]
    for _ in range(3):
        abi.sparda_forecast_select(loop.p, loop.F[0], 1, 1, w.T - 1, loop.kc[1], loop.idx[1],
                                   loop.ws_sel[0])
        abi.sparda_sparse_attn_decode(loop.p, loop.Q[0], kv, kv.view(-1)[w.blk * w.d:], bg,
                                      loop.blk_elems, loop.idx[0], abi.SPARDA_ADDR_LOGICAL,
                                      loop.O[0], loop.ws_att, loop.status)
    torch.cuda.synchronize()
    st = int(loop.status.item())
    print("profile case: B=%d, %d select + %d attention launches, device status %d" % (w.B, 3, 3, st))
    del loop
    torch.cuda.empty_cache()
    # a prefill chunk of 512 tokens of one sequence (0.5 GB of K/V): two
    # passes of its selection (score tiles, row ranking) and attention
    pc = PrefillChunk(W.scaled(W.WORKLOADS["prefill_b4_t128k_c2k"], B=1, nq=512))
    pc.compress()
    for _ in range(2):
        pc.select()
        pc.attention()
    torch.cuda.synchronize()
    st2 = int(pc.status.item())
    print("profile case: prefill B=1, 512 tokens, device status %d" % st2)
    del pc
    torch.cuda.empty_cache()
    # the host gather: one layer of B=2 sequences (1.1 GB of K/V in pinned host
    # memory), two cold gathers of every (b, g)'s 64 top-k blocks (33.5 MB)
    wg = W.scaled(WORKLOAD, B=2, layers=1)
    gl = DecodeLoop(wg, with_host=True)
    for _ in range(2):
        abi.sparda_prefetch_blocks(gl.p, gl.host_kv[0], gl.idx[0], gl.slots[0], True, 0, gl.status)
    # the cached selection into the layer's slot cache (2S slots): cold, then
    # warm (every block a hit)
    gl.setup_cache(2 * wg.S, 0.0, 2)
    for _ in range(2):
        abi.sparda_forecast_select_cached(gl.p, gl.F[0], 1, wg.T - 1, gl.kc[0], gl.idx[0],
                                          gl.ws_sel[0], gl.C, gl.block_of[0], gl.hand[0],
                                          gl.phys[0], gl.fetch[0], gl.host_kv[0], gl.cache[0],
                                          gl.status)
    torch.cuda.synchronize()
    st3 = int(gl.status.item())
    gl.unregister()
    print("profile case: host gather and cached selection B=2, device status %d" % st3)
    del gl
    torch.cuda.empty_cache()
    # the original selector's per-head softmax form at B=16, T=128K: two
    # launches on one layer of block keys (67 MB), then two on window keys
    # (268 MB)
    for windows in (False, True):
        hc = HeadSoftmaxCase(windows, n_layers=1)
        for _ in range(2):
            hc.head_softmax(hc.kc[0])
        torch.cuda.synchronize()
        del hc
        torch.cuda.empty_cache()
    print("profile case: head-softmax selection on block and window keys")
    if st != 0 or st2 != 0 or st3 != 0:
        sys.exit(1)


def run_reference(args):
    """The oracle (plain fp64 CPU code) on the host cores, same metric and
    workload: every step runs the oracle's selection and attention for all 16
    sequences and 4 layers (inputs drawn on the host, K|V only for the blocks
    each layer's sets name)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    w = WORKLOAD
    smp = oracle_sample_synthetic(w, w.seed)
    for _ in range(args.warmup):
        smp.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        smp.step()
    el = time.perf_counter() - t0
    v = w.B * args.steps / el
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "layers": w.layers, "Hq": w.Hq,
                   "G": w.G, "d": w.d, "block": w.blk, "k": w.k, "n_init": w.n_init,
                   "n_local": w.n_local},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": "all %d sequences x %d layers per step (select of every "
                                   "(sequence, group) over %d blocks + attention of every head "
                                   "over its %d-block set); inputs drawn on the host"
                                   % (w.B, w.layers, w.NB, w.S)},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_only(args):
    """One leg alone, on one GPU, its JSON line only (for profiling a leg)."""
    import torch
    from block_sparse_long_sparda_b200 import build
    build.build()
    torch.cuda.set_device(0)
    fn = {"prefill": lambda: run_prefill(args.steps), "sweep": run_sweep,
          "windows": lambda: run_windows(args.steps), "real-model": lambda: run_real_model(args.steps),
          "head-softmax": lambda: run_head_softmax(args.steps)}[args.only]
    out = fn()
    print(json.dumps(out), flush=True)
    if out.get("device_status", 0) != 0:
        sys.exit(1)


def main():
    args = parse_args()
    if args.profile_case:
        from block_sparse_long_sparda_b200 import build
        build.build()
        run_profile_case()
    elif args.impl == "reference":
        run_reference(args)
    elif args.only:
        run_only(args)
    else:
        run_sparda(args)


if __name__ == "__main__":
    main()
