"""Parity at the benchmark's full sizes, in the launch configuration it times.

The decode loop (B=16, T=131072, 4 layers, 34 GB of K/V in HBM) and the
prefill chunk (B=4, T=131072, 2048 query tokens) run exactly as bench.py
runs them -- the same classes, kernels, grids and workspaces.  The oracle
then recomputes a sample of outputs one by one on the host:

- the compressed keys of the sampled (sequence, group) pairs;
- their block sets (same bf16 Kc bytes in, the band rule for near-ties);
- their attention outputs, over the block set the GPU used, so attention
  parity does not depend on the selection.
"""
import os
import sys

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_sparda_b200 import abi, build
from block_sparse_long_sparda_b200 import workloads as W
from tests.parity import check_attention, check_sets, host_bits, pooled_scores_f64, scores_f64

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    abi.lib()
    torch.cuda.init()


def _check_kc_bits(gpu_bits, ora_bits, what):
    same = np.mean(gpu_bits == ora_bits)
    diff = np.abs(gpu_bits.astype(np.int32) - ora_bits.astype(np.int32)).max()
    assert same >= 0.999 and diff <= 1, "%s: bf16 Kc identical %.5f, max diff %d ulp" % (what, same, diff)


def test_decode_loop_full_size_sampled():
    import bench
    w = bench.WORKLOAD
    loop = bench.DecodeLoop(w, with_host=False)
    loop.step_resident()  # select(l -> l+1) beside attention(l), for the four layers
    torch.cuda.synchronize()
    assert int(loop.status.item()) == 0
    L, R, d, blk, NB, T = w.layers, w.r, w.d, w.blk, w.NB, w.T
    rng = np.random.default_rng(2024)
    for l in range(L):
        picks = {(0, 0), (w.B - 1, w.G - 1)}
        while len(picks) < 3:
            picks.add((int(rng.integers(w.B)), int(rng.integers(w.G))))
        if l == 1:  # one layer in full: every (sequence, group)
            picks = {(b, g) for b in range(w.B) for g in range(w.G)}
        for b, g in sorted(picks):
            what = "layer %d b %d g %d" % (l, b, g)
            kv = host_bits(loop.kv[l, b, g])                    # [NB][2][64][128]
            # compressed keys: each block's 64 K rows pooled, as the bench pools them
            _, ora_kc = oracle.compress_keys(kv, blk, shape=(1, NB, blk, d),
                                             strides=(2 * blk * d, d))
            gpu_kc = host_bits(loop.kc[l, b, g])
            _check_kc_bits(gpu_kc, ora_kc.reshape(NB, d), what)
            # the set attention(l) used came from F_{l-1} scoring Kc_l
            F = host_bits(loop.F[(l - 1) % L, b, g]).reshape(1, 1, 1, 1, d)
            kc_in = gpu_kc.reshape(1, 1, NB, d)
            ora_idx, kth, kth1 = oracle.select(F, kc_in, w.k, w.n_init, w.n_local, T - 1, blk)
            gpu_idx = loop.idx[l, b, g].cpu().numpy().reshape(1, 1, 1, -1)
            check_sets(gpu_idx, ora_idx, kth, kth1, scores_f64(F, kc_in), what, q_pos=T - 1,
                       n_init=w.n_init, n_local=w.n_local)
            # attention of the group's heads over the GPU's set
            Q = host_bits(loop.Q[l, b, g * R:(g + 1) * R]).reshape(1, 1, R, d)
            flat = kv.reshape(-1)
            ora_o = oracle.sparse_attention(Q, flat, flat[blk * d:], gpu_idx, T - 1, T, blk,
                                            bg_stride=flat.size, blk_stride=2 * blk * d, G=1)
            gpu_o = host_bits(loop.O[l, b, g * R:(g + 1) * R]).reshape(1, 1, R, d)
            check_attention(gpu_o, ora_o, what)
    del loop
    torch.cuda.empty_cache()


def _check_layer_against_host(loop, l, what, rows_of, pairs=None, QFO=None):
    """Layer l of a host-offload step: its sets against the oracle (F_{l-1}
    scoring Kc_l), the device copy of every set entry byte-exact against the
    oracle's gather from the pinned host bytes, and the attention output over
    the host blocks of the GPU's set.  rows_of(b, g) returns the device copies
    the attention read, in list order ([S][2][64][128] bf16 bits; slot mode:
    slot s, slot cache: slot phys[s]).  QFO: the step's (Q, F, O) device
    tensors when they are not the loop's own."""
    w = loop.w
    L, R, d, blk, NB, T = w.layers, w.r, w.d, w.blk, w.NB, w.T
    idx_all = loop.idx[l].cpu().numpy()
    kc_all = host_bits(loop.kc[l])
    Qd, Fd, Od = QFO if QFO is not None else (loop.Q, loop.F, loop.O)
    F_all = host_bits(Fd[(l - 1) % L])
    Q_all = host_bits(Qd[l])
    O_all = host_bits(Od[l])
    pairs = pairs or [(b, g) for b in range(w.B) for g in range(w.G)]
    for b, g in pairs:
        tag = "%s layer %d b %d g %d" % (what, l, b, g)
        F = F_all[b, g].reshape(1, 1, 1, 1, d)
        kc_in = kc_all[b, g].reshape(1, 1, NB, d)
        ora_idx, kth, kth1 = oracle.select(F, kc_in, w.k, w.n_init, w.n_local, T - 1, blk)
        gpu_idx = idx_all[b, g].reshape(1, 1, 1, -1)
        check_sets(gpu_idx, ora_idx, kth, kth1, scores_f64(F, kc_in), tag, q_pos=T - 1,
                   n_init=w.n_init, n_local=w.n_local)
        host = loop.host_kv[l, b, g].view(torch.int16).numpy().view(np.uint16)  # [NB][2][64][128]
        ids = gpu_idx.reshape(-1)
        want = oracle.gather_blocks(host.reshape(1, 1, NB, 2, blk, d), ids.reshape(1, 1, -1),
                                    T - 1, w.n_init, w.n_local, False)[0, 0]
        got = rows_of(b, g)
        for s_ in range(len(ids)):
            if ids[s_] >= 0:
                assert np.array_equal(got[s_], want[s_]), "%s: entry %d (block %d)" % (tag, s_, ids[s_])
        Q = Q_all[b, g * R:(g + 1) * R].reshape(1, 1, R, d)
        flat = host.reshape(-1)
        ora_o = oracle.sparse_attention(Q, flat, flat[blk * d:], gpu_idx, T - 1, T, blk,
                                        bg_stride=flat.size, blk_stride=2 * blk * d, G=1)
        check_attention(O_all[b, g * R:(g + 1) * R].reshape(1, 1, R, d), ora_o, tag)


def test_offload_loop_full_size():
    """The decode loop as bench.py's e2e legs run it, at full size: the K/V
    of all four layers in pinned host memory (32 GiB).  One cold step -- per
    layer the next layer's blocks are selected, gathered over the host link
    into device slots on a side stream while this layer attends from its own
    slots -- then three steps through the device slot cache (one launch
    selecting, planning and fetching the misses only, on a high-priority
    stream; attention reading each entry from its cache slot; inputs
    uploaded and outputs sent back on a copy stream) with drifting Forecast
    vectors.  After each step, every (sequence, group) of
    the layers whose sets and slots are still those the step attended over
    (layers 1-3; layer 0's were replaced for the next step) is checked
    against the oracle: sets, device copies byte for byte against the host
    bytes, and outputs."""
    import bench
    w = bench.WORKLOAD
    loop = bench.DecodeLoop(w, with_host=True)
    try:
        loop.step_e2e()
        torch.cuda.synchronize()
        assert int(loop.status.item()) == 0
        for l in range(1, w.layers):
            _check_layer_against_host(loop, l, "slots",
                                      lambda b, g, l=l: host_bits(loop.slots[l, b, g]))
        loop.setup_cache(2 * w.S, 0.01, 4)
        loop.prime_cache()
        loop.begin_cached(0)
        fetched = []
        for t in range(3):
            loop.step_e2e_cached(t)
            torch.cuda.synchronize()
            assert int(loop.status.item()) == 0
            fetched.append(int(loop.fetch[1:].sum().item()))
            phys = torch.from_numpy(np.maximum(loop.phys.cpu().numpy(), 0)).long().cuda()
            pairs = [(b, g) for b in range(w.B) for g in range(w.G)] if t == 2 else \
                [(0, 0), (w.B - 1, w.G - 1), (5, 3)]
            for l in range(1, w.layers):
                _check_layer_against_host(
                    loop, l, "cache step %d" % t,
                    lambda b, g, l=l: host_bits(loop.cache[l, b, g].index_select(0, phys[l, b, g])),
                    pairs=pairs, QFO=loop.step_inputs(t))
            # the outputs that went back to the host are the step's
            assert torch.equal(loop.h_out.view(torch.int16),
                               loop.step_inputs(t)[2].cpu().view(torch.int16))
        # drifting sets: later steps fetch only a few blocks, never the whole set
        assert fetched[-1] < 0.1 * (w.layers - 1) * w.B * w.G * w.k, fetched
    finally:
        loop.unregister()
        del loop
        torch.cuda.empty_cache()


def test_real_model_decode_loop_full_size_sampled():
    """The real models' decode configuration as bench.py times it: 96-block
    sets on the window grid, 16 sequences of mixed lengths.  Each sample's
    set is checked against the oracle run on that sequence alone (its own
    length and query position), and its attention over the GPU's set."""
    import bench
    w = W.WORKLOADS["decode_loop_b16_t128k_budget96"]
    loop = bench.DecodeLoop(w, with_host=False)
    loop.step_resident()
    torch.cuda.synchronize()
    assert int(loop.status.item()) == 0
    L, R, d, blk = w.layers, w.r, w.d, w.blk
    rng = np.random.default_rng(2026)
    shortest = int(np.argmin(loop.lens))
    for l in range(L):
        picks = {(shortest, 0), (w.B - 1, w.G - 1)}
        while len(picks) < 3:
            picks.add((int(rng.integers(w.B)), int(rng.integers(w.G))))
        for b, g in sorted(picks):
            Lb = int(loop.lens[b])
            what = "layer %d b %d g %d (length %d)" % (l, b, g, Lb)
            nw = oracle.window_count(Lb)
            kw = np.ascontiguousarray(host_bits(loop.kw[l, b, g])[:nw]).reshape(1, 1, nw, d)
            F = host_bits(loop.F[(l - 1) % L, b, g]).reshape(1, 1, 1, 1, d)
            ora_idx, kth, kth1 = oracle.select_windows(F, kw, Lb, w.k, w.n_init, w.n_local, Lb - 1)
            gpu_idx = loop.idx[l, b, g].cpu().numpy().reshape(1, 1, 1, -1)
            assert gpu_idx.shape[-1] == 96
            check_sets(gpu_idx, ora_idx, kth, kth1,
                       pooled_scores_f64(F, kw, (Lb + blk - 1) // blk), what, q_pos=Lb - 1,
                       n_init=w.n_init, n_local=w.n_local)
            kv = host_bits(loop.kv[l, b, g])
            Q = host_bits(loop.Q[l, b, g * R:(g + 1) * R]).reshape(1, 1, R, d)
            flat = kv.reshape(-1)
            ora_o = oracle.sparse_attention(Q, flat, flat[blk * d:], gpu_idx, Lb - 1, Lb, blk,
                                            bg_stride=flat.size, blk_stride=2 * blk * d, G=1)
            gpu_o = host_bits(loop.O[l, b, g * R:(g + 1) * R]).reshape(1, 1, R, d)
            check_attention(gpu_o, ora_o, what)
    del loop
    torch.cuda.empty_cache()


def test_decode_large_batch_multiwave_sampled():
    """A decode batch large enough that the attention's list entries need
    more CTAs than one wave holds (B = 128: 68,608 entries, at most 128 per
    CTA) and the selection runs 1024 single-chunk problems: compression,
    selection and attention on the device, sampled pairs against the oracle."""
    B, G, R, T, d, k = 128, 8, 4, 8192, 128, 64
    NB = T // 64
    S = k + 3
    dev = torch.device("cuda")
    K = torch.empty(B, G, T, d, dtype=torch.bfloat16, device=dev)
    V = torch.empty(B, G, T, d, dtype=torch.bfloat16, device=dev)
    W.torch_normal_bf16_(K, 9001)
    W.torch_normal_bf16_(V, 9002)
    gen = torch.Generator(device=dev)
    gen.manual_seed(9003)
    Q = torch.randn(B, G * R, d, generator=gen, device=dev).to(torch.bfloat16)
    F = torch.randn(B, G, d, generator=gen, device=dev).to(torch.bfloat16)
    p = abi.make_params(B, G * R, G, T, k)
    kc = torch.empty(B, G, NB, d, dtype=torch.bfloat16, device=dev)
    abi.sparda_compress_keys(p, K, T * d, d, None, kc)
    idx = torch.full((B, G, S), -7, dtype=torch.int32, device=dev)
    abi.sparda_forecast_select(p, F, 1, 1, T - 1, kc, idx, abi.workspace(abi.SPARDA_OP_SELECT, p, 1, 1))
    O = torch.empty(B, G * R, d, dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    abi.sparda_sparse_attn_decode(p, Q, K, V, T * d, 64 * d, idx, 0, O,
                                  abi.workspace(abi.SPARDA_OP_ATTN_DECODE, p), status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rng = np.random.default_rng(2027)
    picks = {(0, 0), (B - 1, G - 1), (B // 2, 3)}
    while len(picks) < 6:
        picks.add((int(rng.integers(B)), int(rng.integers(G))))
    for b, g in sorted(picks):
        what = "B=128 b %d g %d" % (b, g)
        Kb = host_bits(K[b, g]).reshape(1, 1, T, d)
        _, ora_kc = oracle.compress_keys(Kb)
        gpu_kc = host_bits(kc[b, g]).reshape(1, 1, NB, d)
        _check_kc_bits(gpu_kc.reshape(NB, d), ora_kc.reshape(NB, d), what)
        Fb = host_bits(F[b, g]).reshape(1, 1, 1, 1, d)
        ora_idx, kth, kth1 = oracle.select(Fb, gpu_kc, k, 1, 2, T - 1)
        gpu_idx = idx[b, g].cpu().numpy().reshape(1, 1, 1, -1)
        check_sets(gpu_idx, ora_idx, kth, kth1, scores_f64(Fb, gpu_kc), what, q_pos=T - 1,
                   n_init=1, n_local=2)
        Qb = host_bits(Q[b, g * R:(g + 1) * R]).reshape(1, 1, R, d)
        Vb = host_bits(V[b, g]).reshape(1, 1, T, d)
        ora_o = oracle.sparse_attention(Qb, Kb, Vb, gpu_idx, T - 1, T)
        check_attention(host_bits(O[b, g * R:(g + 1) * R]).reshape(1, 1, R, d), ora_o, what)
    del K, V
    torch.cuda.empty_cache()


def test_prefill_chunk_full_size_sampled():
    import bench
    pc = bench.PrefillChunk()
    w = pc.w
    pc.compress()
    pc.select()
    pc.attention()
    torch.cuda.synchronize()
    assert int(pc.status.item()) == 0
    R, d, blk, NB, T, q0 = w.r, w.d, w.blk, w.NB, w.T, pc.q0
    rng = np.random.default_rng(2025)
    # the first and last query tokens, the two sides of a block boundary, and
    # random ones
    first_of_block = (64 - q0 % 64) % 64 or 64
    tokens = {0, w.nq - 1, first_of_block - 1, first_of_block}
    picks = set()
    for i in tokens:
        picks.add((int(rng.integers(w.B)), i, int(rng.integers(w.G))))
    while len(picks) < 7:
        picks.add((int(rng.integers(w.B)), int(rng.integers(w.nq)), int(rng.integers(w.G))))
    kc_cache = {}
    for b, i, g in sorted(picks):
        what = "b %d token %d g %d" % (b, i, g)
        K = host_bits(pc.K[b, g]).reshape(1, 1, T, d)
        V = host_bits(pc.V[b, g]).reshape(1, 1, T, d)
        if (b, g) not in kc_cache:
            _, ora_kc = oracle.compress_keys(K, blk)
            gpu_kc = host_bits(pc.kc[b, g])
            _check_kc_bits(gpu_kc, ora_kc.reshape(NB, d), "b %d g %d" % (b, g))
            kc_cache[(b, g)] = gpu_kc.reshape(1, 1, NB, d)
        kc_in = kc_cache[(b, g)]
        F = host_bits(pc.F[b, i, g]).reshape(1, 1, 1, 1, d)
        ora_idx, kth, kth1 = oracle.select(F, kc_in, w.k, w.n_init, w.n_local, q0 + i, blk)
        gpu_idx = pc.idx[b, i, g].cpu().numpy().reshape(1, 1, 1, -1)
        check_sets(gpu_idx, ora_idx, kth, kth1, scores_f64(F, kc_in), what, q_pos=q0 + i,
                   n_init=w.n_init, n_local=w.n_local)
        Q = host_bits(pc.Q[b, i, g * R:(g + 1) * R]).reshape(1, 1, R, d)
        ora_o = oracle.sparse_attention(Q, K, V, gpu_idx, q0 + i, T, blk)
        gpu_o = host_bits(pc.O[b, i, g * R:(g + 1) * R]).reshape(1, 1, R, d)
        check_attention(gpu_o, ora_o, what)
    # every row of the chunk: the listed-threshold ranking against the full
    # binned search on the same score keys (both exact, so bit for bit)
    p_full = abi.make_params(w.B, w.Hq, w.G, T, w.k, w.n_init, w.n_local,
                             tune={"select_binned": 1})
    idx_full = torch.full_like(pc.idx, -7)
    abi.sparda_forecast_select(p_full, pc.F, w.nq, 1, q0, pc.kc, idx_full, pc.ws_sel, pc.status)
    torch.cuda.synchronize()
    assert int(pc.status.item()) == 0
    assert torch.equal(idx_full, pc.idx), "%d of %d rows differ" % (
        int((idx_full != pc.idx).any(dim=-1).sum()), w.B * w.nq * w.G)
    del pc
    torch.cuda.empty_cache()


@pytest.mark.parametrize("windows", [False, True])
def test_head_softmax_full_size(windows):
    """The original selector's per-head softmax form at the shapes bench.py
    times (B=16, G=8 groups of 4 query heads, T=131072, k=64 + 1 initial +
    2 local), through the same class: every (sequence, group) set against the
    oracle on the same key bytes."""
    import bench
    c = bench.HeadSoftmaxCase(windows, n_layers=1)
    c.head_softmax(c.kc[0])
    torch.cuda.synchronize()
    got = c.idx.cpu().numpy()
    w = c.w
    Q, kc = host_bits(c.Q), host_bits(c.kc[0])
    ora, kth, kth1, wb = oracle.select_head_softmax(Q, kc, w.T, w.k, w.n_init, w.n_local, w.T - 1,
                                                    c.tau, windows=windows)
    B, G, S = got.shape
    exact = check_sets(got.reshape(B, 1, G, S), ora.reshape(B, 1, G, S), kth.reshape(B, 1, G),
                       kth1.reshape(B, 1, G), wb.reshape(B, 1, G, -1), "head softmax full size",
                       q_pos=w.T - 1, n_init=w.n_init, n_local=w.n_local)
    assert exact >= B * G - 2, "only %d of %d sets bit-exact" % (exact, B * G)
