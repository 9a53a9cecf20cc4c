"""GPU parity: every entry point of libsparda, called through the C ABI, against
the fp64 CPU oracle on the same seeded inputs, at sizes the oracle finishes in
seconds that still span several thread blocks and a ragged tail, plus the
degenerate cases of the method."""
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_sparda_b200 import abi, build
from block_sparse_long_sparda_b200 import workloads as W
from tests.parity import (Guarded, bf16_f64, check_attention, check_compressed, check_sets,
                          dev_bf16, guarded_workspace, host_bits, pooled_scores_f64, scores_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    abi.lib()
    torch.cuda.init()


def gpu_compress(K_bits, blk=64):
    B, G, T, d = K_bits.shape
    p = abi.make_params(B, G, G, T, 1)
    K = dev_bf16(K_bits)
    NB = (T + blk - 1) // blk
    kc32 = Guarded((B, G, NB, d), torch.float32)
    kc16 = Guarded((B, G, NB, d), torch.bfloat16)
    abi.sparda_compress_keys(p, K, T * d, d, kc32.t, kc16.t)
    return kc32.check("fp32 Kc").cpu().numpy(), host_bits(kc16.check("bf16 Kc"))


def gpu_select(F_bits, kc_bits, k, n_init, n_local, q_start, T, Hq=None, tune=None):
    """F [B][nq][G][nf][d] bits, kc [B][G][NB][d] bits -> idx [B][nq][G][S].
    tune: optional sparda_tuning fields (forces a kernel variant)."""
    B, nq, G, nf, d = F_bits.shape
    p = abi.make_params(B, Hq or G * max(nf, 1), G, T, k, n_init, n_local, tune=tune)
    S = k + n_init + n_local
    idx = Guarded((B, nq, G, S), torch.int32, fill=-7)
    ws = guarded_workspace(abi.SPARDA_OP_SELECT, p, nq, nf)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.sparda_forecast_select(p, dev_bf16(F_bits), nq, nf, q_start, dev_bf16(kc_bits), idx.t,
                               ws and ws.t, status)
    out = idx.check("block sets").cpu().numpy()
    if ws is not None:
        ws.check("select workspace")
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    assert not (out == -7).any(), "entries left unwritten"
    return out


def gpu_decode(Q_bits, K_bits, V_bits, idx, T, k, n_init=1, n_local=2, addr_mode=0,
               bg_stride=None, blk_stride=None, status=None, tune=None):
    B, Hq, d = Q_bits.shape
    G = idx.shape[1]
    p = abi.make_params(B, Hq, G, T, k, n_init, n_local, tune=tune)
    K = dev_bf16(K_bits)
    V = dev_bf16(V_bits) if V_bits is not None else None
    if bg_stride is None:
        bg_stride, blk_stride = K_bits.shape[2] * d, 64 * d
    O = Guarded((B, Hq, d), torch.bfloat16)
    ws = guarded_workspace(abi.SPARDA_OP_ATTN_DECODE, p)
    didx = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda()
    if V is None:  # interleaved storage: V rows follow the K rows of each block
        V = K.view(-1)[64 * d:]
    abi.sparda_sparse_attn_decode(p, dev_bf16(Q_bits), K, V, bg_stride, blk_stride, didx,
                                  addr_mode, O.t, ws and ws.t, status)
    out = host_bits(O.check("attention output"))
    if ws is not None:
        ws.check("attention workspace")
    return out


# --------------------------------------------------------------------------
# compressed keys
# --------------------------------------------------------------------------

@pytest.mark.parametrize("T", [4096, 4096 + 37, 64, 1])
def test_compress_parity(T):
    rng = W.rng_for(7, T)
    K = W.normal_bf16(rng, (2, 3, T, 128))
    kc32, kc16 = gpu_compress(K)
    ora, orab = oracle.compress_keys(K)
    check_compressed(kc32, kc16, ora, orab)


def test_compress_decode_b4_t32k_planted():
    w = W.WORKLOADS["decode_b4_t32k_planted"]
    x = W.decode_inputs(w)
    kc32, kc16 = gpu_compress(x["K"])
    ora, orab = oracle.compress_keys(x["K"])
    check_compressed(kc32, kc16, ora, orab)


def test_compress_strided_rows():
    rng = W.rng_for(8)
    B, G, T, d = 1, 2, 300, 128
    big = W.normal_bf16(rng, (B, G, T, 2 * d))          # each token row padded to 2d
    p = abi.make_params(B, G, G, T, 1)
    kc32 = torch.empty(B, G, 5, d, dtype=torch.float32, device="cuda")
    abi.sparda_compress_keys(p, dev_bf16(big), T * 2 * d, 2 * d, kc32, None)
    torch.cuda.synchronize()
    ora, _ = oracle.compress_keys(np.ascontiguousarray(big[..., :d]))
    assert np.abs(kc32.cpu().numpy() - ora).max() <= 1e-3


# --------------------------------------------------------------------------
# selection
# --------------------------------------------------------------------------

def _select_case(F, kc, k, n_init, n_local, q_start, T, what, tune=None):
    ora, kth, kth1 = oracle.select(F, kc, k, n_init, n_local, q_start)
    got = gpu_select(F, kc, k, n_init, n_local, q_start, T, tune=tune)
    nq = F.shape[1]
    return check_sets(got, ora, kth, kth1, scores_f64(F, kc), what,
                      q_pos=q_start + np.arange(nq)[None, :], n_init=n_init, n_local=n_local)


@pytest.mark.parametrize("name", ["decode_b1_t4k", "decode_b4_t32k_planted"])
def test_select_decode_configs(name):
    w = W.WORKLOADS[name]
    x = W.decode_inputs(w)
    _, kcb = oracle.compress_keys(x["K"])
    F = x["F"].reshape(w.B, 1, w.G, 1, w.d)
    _select_case(F, kcb, w.k, w.n_init, w.n_local, w.T - 1, w.T, name)


@pytest.mark.parametrize("NB,B", [(128, 1), (2048, 16), (16384, 1), (16384, 4), (1000, 3)])
def test_select_sweep_points(NB, B):
    x = W.sweep_inputs(NB, B)
    F = x["F"].reshape(B, 1, 8, 1, 128)
    _select_case(F, x["kc"], 64, 1, 2, NB * 64 - 1, NB * 64, "sweep NB=%d B=%d" % (NB, B))


@pytest.mark.parametrize("chunk", ["256", "512", "8192"])
def test_select_forced_chunking(chunk):
    x = W.sweep_inputs(3000, 2)
    F = x["F"].reshape(2, 1, 8, 1, 128)
    _select_case(F, x["kc"], 64, 1, 2, 3000 * 64 - 1, 3000 * 64, "chunk " + chunk,
                 tune={"select_chunk": int(chunk)})


def test_select_baseline_multihead():
    x = W.sweep_inputs(2048, 2)
    Qg = x["Q"].reshape(2, 1, 8, 4, 128)                 # 4 query heads per group, summed
    _select_case(Qg, x["kc"], 64, 1, 2, 2048 * 64 - 1, 2048 * 64, "baseline")


@pytest.mark.parametrize("k", [100, 64, 17, 1])
@pytest.mark.parametrize("binned", [False, True])
@pytest.mark.parametrize("chunk", ["0", "256"])
def test_select_exact_ties_lower_index_wins(chunk, binned, k):
    # k <= 64 over at most 2048 candidates takes the sorting-network threshold
    # unless the binned search is forced; both must give the oracle's sets
    tune = {"select_chunk": int(chunk), "select_binned": int(binned)}
    rng = np.random.default_rng(3)
    NB, B, G, d = 1500, 2, 4, 128
    kc = np.zeros((B, G, NB, d), np.float32)
    kc[..., 0] = rng.integers(-3, 4, size=(B, G, NB))     # many exact ties
    F = np.zeros((B, 1, G, 1, d), np.float32)
    F[..., 0] = 1.0
    Fb, kcb = W.f32_to_bf16_bits(F), W.f32_to_bf16_bits(kc)
    ora, _, _ = oracle.select(Fb, kcb, k, 1, 2, NB * 64 - 1)
    got = gpu_select(Fb, kcb, k, 1, 2, NB * 64 - 1, NB * 64, tune=tune)
    assert np.array_equal(got, ora)


@pytest.mark.parametrize("k,n_init,n_local", [(0, 1, 2), (61, 1, 2), (70, 1, 2), (5, 0, 0),
                                              (5, 3, 7), (1, 0, 1)])
def test_select_degenerate_budgets(k, n_init, n_local):
    rng = W.rng_for(11, k * 100 + n_init * 10 + n_local)
    NB, B, G = 64, 2, 2
    kc = W.normal_bf16(rng, (B, G, NB, 128))
    F = W.normal_bf16(rng, (B, 1, G, 1, 128))
    _select_case(F, kc, k, n_init, n_local, NB * 64 - 1, NB * 64, "budget")


@pytest.mark.parametrize("T", [1, 63, 64, 65, 130, 4096 + 17])
def test_select_short_and_ragged_sequences(T):
    rng = W.rng_for(12, T)
    NB = (T + 63) // 64
    kc = W.normal_bf16(rng, (1, 2, NB, 128))
    F = W.normal_bf16(rng, (1, 1, 2, 1, 128))
    _select_case(F, kc, 4, 1, 2, T - 1, T, "T=%d" % T)


def test_select_prefill_chunk():
    rng = W.rng_for(13)
    B, G, T, nq = 2, 4, 8192, 96
    NB = T // 64
    kc = W.normal_bf16(rng, (B, G, NB, 128))
    F = W.normal_bf16(rng, (B, nq, G, 1, 128))
    _select_case(F, kc, 16, 1, 2, T - nq, T, "prefill")
    # a chunk that starts inside the first blocks (short candidate lists)
    _select_case(F, kc, 16, 1, 2, 0, T, "prefill from 0")


@pytest.mark.parametrize("T,nq,q_off,k", [(40000 + 37, 200, 0, 64), (20000, 130, 7000, 100),
                                           (8192, 64, 0, 1), (16384 + 64, 300, 3000, 512),
                                           (200000 + 5, 64, 0, 64)])
def test_select_prefill_tensor_scores(T, nq, q_off, k):
    """Chunks scored on the tensor cores: several 256-block tiles, a ragged
    last block, partial 128-token tiles, chunks ending before the sequence
    does, budgets from 1 to 512, and rows longer than the 2048 keys a warp
    holds in registers."""
    rng = W.rng_for(17 + T)
    B, G = 2, 3
    NB = (T + 63) // 64
    kc = W.normal_bf16(rng, (B, G, NB, 128))
    F = W.normal_bf16(rng, (B, nq, G, 1, 128))
    _select_case(F, kc, k, 1, 2, T - nq - q_off, T, "prefill tensor")


@pytest.mark.parametrize("k", [1, 17, 64, 300])
def test_select_prefill_exact_ties_lower_index_wins(k):
    """The row ranking of the tensor-core prefill path (>= 64 query tokens)
    on integer scores: runs of exactly equal keys at the threshold, rows
    whose threshold bin is one key, and rows keeping only some of the keys
    equal to the k-th; the lower block index must win every tie, as in the
    oracle.  Some tokens score with the opposite sign, so both ends of the
    key range are ranked."""
    rng = np.random.default_rng(5 + k)
    NB, B, G, nq = 1500, 1, 2, 96
    T = NB * 64
    kc = np.zeros((B, G, NB, 128), np.float32)
    kc[..., 0] = rng.integers(-3, 4, size=(B, G, NB))
    F = np.zeros((B, nq, G, 1, 128), np.float32)
    F[..., 0] = np.where(rng.random((B, nq, G, 1)) < 0.5, 1.0, -1.0)
    Fb, kcb = W.f32_to_bf16_bits(F), W.f32_to_bf16_bits(kc)
    ora, _, _ = oracle.select(Fb, kcb, k, 1, 2, T - nq)
    got = gpu_select(Fb, kcb, k, 1, 2, T - nq, T)
    assert np.array_equal(got, ora)


def _exact_score_case(rng, B, G, NB, nq, pattern):
    """Forecast vectors and compressed keys whose scores are exact in bf16
    products and fp32 sums: score = a + b / 256 with integer a, b in
    [-128, 128] (F = (+-1, +-1/256, 0, ...)), so the device keys and the
    oracle's fp64 scores order the blocks identically and the sets must match
    bit for bit."""
    kc = np.zeros((B, G, NB, 128), np.float32)
    a = rng.integers(-128, 129, size=(B, G, NB))
    b = rng.integers(-128, 129, size=(B, G, NB))
    if pattern == "lane":  # one lane's entries (block 1 + 32 m + 5) all score high
        a[..., 6::32] = rng.integers(100, 129, size=a[..., 6::32].shape)
    elif pattern == "outlier":  # one far outlier: every other listed key shares a bin
        a[...] = rng.integers(0, 2, size=a.shape)
        a[..., NB // 2] = 128
    elif pattern == "ties":  # few distinct values: ties straddle the k-th
        a[...] = rng.integers(0, 4, size=a.shape)
        b[...] = 0
    kc[..., 0], kc[..., 1] = a, b
    F = np.zeros((B, nq, G, 1, 128), np.float32)
    sgn = np.where(rng.random((B, nq, G, 1)) < 0.8, 1.0, -1.0)
    F[..., 0] = sgn
    F[..., 1] = sgn / 256.0
    return W.f32_to_bf16_bits(F), W.f32_to_bf16_bits(kc)


@pytest.mark.parametrize("k", [1, 8, 33, 64])
@pytest.mark.parametrize("pattern", ["random", "lane", "outlier", "ties"])
def test_select_prefill_listed_threshold_exact(k, pattern):
    """The row ranking's listed threshold (k <= 64, rows of 1024-2048 keys)
    and every way it hands a row to the full search -- a lane listing more
    keys than it holds, a threshold bin of more than 32 keys, keys equal to
    the k-th only partly kept -- on exactly representable scores: the sets
    equal the oracle's bit for bit, and those of the full search on every
    row (select_binned)."""
    rng = np.random.default_rng(23 + 7 * k + len(pattern))
    B, G, NB, nq = 1, 2, 2048, 96
    T = NB * 64
    Fb, kcb = _exact_score_case(rng, B, G, NB, nq, pattern)
    ora, _, _ = oracle.select(Fb, kcb, k, 1, 2, T - nq)
    got = gpu_select(Fb, kcb, k, 1, 2, T - nq, T)
    assert np.array_equal(got, ora), pattern
    full = gpu_select(Fb, kcb, k, 1, 2, T - nq, T, tune={"select_binned": 1})
    assert np.array_equal(full, ora), pattern


def test_select_prefill_listed_threshold_short_rows():
    """Rows of 1024 keys, the shortest the listed threshold takes, next to
    rows just below it, which the full search ranks."""
    rng = np.random.default_rng(31)
    B, G, NB, nq = 1, 2, 1027, 96
    T = NB * 64
    Fb, kcb = _exact_score_case(rng, B, G, NB, nq, "random")
    for k in (16, 64):
        ora, _, _ = oracle.select(Fb, kcb, k, 1, 2, T - nq)
        assert np.array_equal(gpu_select(Fb, kcb, k, 1, 2, T - nq, T), ora)


def test_select_prefill_tensor_matches_streaming_path():
    """The same chunk through both selection paths gives the same sets."""
    rng = W.rng_for(19)
    B, G, T, nq = 1, 2, 24576, 160
    kc = W.normal_bf16(rng, (B, G, T // 64, 128))
    F = W.normal_bf16(rng, (B, nq, G, 1, 128))
    a = gpu_select(F, kc, 64, 1, 2, T - nq, T)
    b = gpu_select(F, kc, 64, 1, 2, T - nq, T, tune={"select_stream": 1})
    ora, kth, kth1 = oracle.select(F, kc, 64, 1, 2, T - nq)
    sc = scores_f64(F, kc)
    qp = T - nq + np.arange(nq)[None, :]
    check_sets(a, ora, kth, kth1, sc, "tensor path", q_pos=qp, n_init=1, n_local=2)
    check_sets(b, ora, kth, kth1, sc, "streaming path", q_pos=qp, n_init=1, n_local=2)


# --------------------------------------------------------------------------
# the window grid (32-token windows at stride 16, max-pooled to blocks)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("T", [31, 32, 1000, 4096 + 37])
def test_compress_windows_parity(T):
    rng = W.rng_for(60 + T)
    B, G, d = 2, 3, 128
    K = W.normal_bf16(rng, (B, G, T, d))
    NW = oracle.window_count(T)
    p = abi.make_params(B, G, G, T, 1)
    kw32 = torch.zeros(B, G, max(NW, 1), d, dtype=torch.float32, device="cuda")
    kw16 = torch.zeros(B, G, max(NW, 1), d, dtype=torch.bfloat16, device="cuda")
    abi.sparda_compress_windows(p, dev_bf16(K), T * d, d, 32, 16, kw32, kw16)
    torch.cuda.synchronize()
    o64, o16 = oracle.compress_windows(K)
    if NW:
        check_compressed(kw32.cpu().numpy()[:, :, :NW], host_bits(kw16)[:, :, :NW], o64, o16)


def _select_windows_case(F, kw, T, k, n_init, n_local, q_start, what, tune=None):
    B, nq, G, nf, d = F.shape
    p = abi.make_params(B, G * nf, G, T, k, n_init, n_local, tune=tune)
    S = k + n_init + n_local
    idx = Guarded((B, nq, G, S), torch.int32, fill=-7)
    ws = guarded_workspace(abi.SPARDA_OP_SELECT_WINDOWS, p, nq, nf)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.sparda_forecast_select_windows(p, dev_bf16(F), nq, nf, q_start, dev_bf16(kw), 32, 16,
                                       idx.t, ws and ws.t, status)
    got = idx.check("window block sets").cpu().numpy()
    if ws is not None:
        ws.check("window select workspace")
    assert int(status.item()) == 0
    assert not (got == -7).any()
    ora, kth, kth1 = oracle.select_windows(F, kw, T, k, n_init, n_local, q_start)
    NB = (T + 63) // 64
    return check_sets(got, ora, kth, kth1, pooled_scores_f64(F, kw, NB), what,
                      q_pos=q_start + np.arange(nq)[None, :], n_init=n_init, n_local=n_local)


@pytest.mark.parametrize("T,k,n_local,chunk", [(8192 + 20, 16, 2, "0"), (32768, 64, 2, "256"),
                                                (5000 + 33, 8, 0, "0"), (20000, 40, 1, "512")])
def test_select_windows_decode(T, k, n_local, chunk):
    rng = W.rng_for(70 + T)
    B, G, d = 2, 3, 128
    kw = W.normal_bf16(rng, (B, G, oracle.window_count(T), d))
    F = W.normal_bf16(rng, (B, 1, G, 1, d))
    _select_windows_case(F, kw, T, k, 1, n_local, T - 1, "windows decode",
                         tune={"select_chunk": int(chunk)})


@pytest.mark.parametrize("T,nq,q_off", [(16384 + 40, 96, 0), (40000, 200, 3000),
                                         (2048 * 64 + 40, 96, 0)])
def test_select_windows_prefill_tensor_path(T, nq, q_off):
    """The last case has 2045-2046 candidates per token: its rows take the
    listed threshold, and must equal the full search's bit for bit."""
    rng = W.rng_for(80 + T)
    B, G, d = 2, 2, 128
    kw = W.normal_bf16(rng, (B, G, oracle.window_count(T), d))
    F = W.normal_bf16(rng, (B, nq, G, 1, d))
    _select_windows_case(F, kw, T, 32, 1, 2, T - nq - q_off, "windows prefill")
    if T > 2048 * 64:
        sets = []
        for tune in (None, {"select_binned": 1}):
            p = abi.make_params(B, G, G, T, 32, 1, 2, tune=tune)
            idx = torch.full((B, nq, G, 35), -7, dtype=torch.int32, device="cuda")
            abi.sparda_forecast_select_windows(
                p, dev_bf16(F), nq, 1, T - nq - q_off, dev_bf16(kw), 32, 16, idx,
                abi.workspace(abi.SPARDA_OP_SELECT_WINDOWS, p, nq, 1))
            sets.append(idx.cpu())
        assert torch.equal(sets[0], sets[1])


def test_select_windows_compressed_from_keys():
    """The chain a caller runs: compress a sequence into windows, then select."""
    rng = W.rng_for(90)
    B, G, T, d = 1, 2, 6000, 128
    K = W.normal_bf16(rng, (B, G, T, d))
    p = abi.make_params(B, G, G, T, 12)
    NW = oracle.window_count(T)
    kw16 = torch.zeros(B, G, NW, d, dtype=torch.bfloat16, device="cuda")
    abi.sparda_compress_windows(p, dev_bf16(K), T * d, d, 32, 16, None, kw16)
    torch.cuda.synchronize()
    F = W.normal_bf16(rng, (B, 1, G, 1, d))
    _select_windows_case(F, host_bits(kw16), T, 12, 1, 2, T - 1, "compressed windows")


# --------------------------------------------------------------------------
# the original selector's per-head softmax form (block and window grids)
# --------------------------------------------------------------------------

def gpu_head_softmax(Q_bits, kc_bits, T, k, n_init, n_local, q_start, tau, windows, lens=None,
                     ws=None, tune=None):
    """Q [B][G][nf][d] bits; kc block or window keys -> idx [B][G][S]."""
    B, G, nf, d = Q_bits.shape
    sl = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = abi.make_params(B, G * nf, G, T, k, n_init, n_local, seq_len=sl, tune=tune)
    S = k + n_init + n_local
    idx = Guarded((B, G, S), torch.int32, fill=-7)
    op = abi.SPARDA_OP_HEAD_SOFTMAX_WINDOWS if windows else abi.SPARDA_OP_HEAD_SOFTMAX
    gws = None
    if ws is None:
        gws = guarded_workspace(op, p, 1, nf)
        ws = gws and gws.t
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if windows:
        abi.sparda_head_softmax_select_windows(p, dev_bf16(Q_bits), nf, q_start, tau,
                                               dev_bf16(kc_bits), 32, 16, idx.t, ws, status)
    else:
        abi.sparda_head_softmax_select(p, dev_bf16(Q_bits), nf, q_start, tau, dev_bf16(kc_bits),
                                       idx.t, ws, status)
    out = idx.check("head-softmax block sets").cpu().numpy()
    if gws is not None:
        gws.check("head-softmax workspace")
    st = int(status.item())
    if lens is None or all(1 <= x <= T for x in lens):
        assert st == 0, "device status %d" % st
    else:
        assert abi.sparda_status_from_device(st) == abi.SPARDA_ERANGE
    assert not (out == -7).any(), "entries left unwritten"
    return out


def _hsm_check(got, Q, kc, T, k, n_init, n_local, q_start, tau, windows, what):
    """got [B][G][S] against the oracle on the same inputs (band rule at near
    ties, on the oracle's own block weights)."""
    ora, kth, kth1, wb = oracle.select_head_softmax(Q, kc, T, k, n_init, n_local, q_start, tau,
                                                    windows=windows)
    B, G, S = got.shape
    return check_sets(got.reshape(B, 1, G, S), ora.reshape(B, 1, G, S), kth.reshape(B, 1, G),
                      kth1.reshape(B, 1, G), wb.reshape(B, 1, G, -1), what, q_pos=q_start,
                      n_init=n_init, n_local=n_local)


@pytest.mark.parametrize("T,nf,k,n_local,chunk", [
    (8192 + 20, 4, 16, 2, "0"), (32768, 4, 64, 2, "256"), (20000, 8, 40, 1, "512"),
    (5000 + 33, 16, 8, 0, "0"), (32768, 2, 100, 2, "0"), (65536 + 64, 4, 63, 32, "0"),
    (12000, 1, 20, 2, "0")])
@pytest.mark.parametrize("windows", [False, True])
def test_head_softmax_select(T, nf, k, n_local, chunk, windows):
    rng = W.rng_for(140 + T + nf, int(windows))
    B, G, d = 2, 3, 128
    NR = oracle.window_count(T) if windows else (T + 63) // 64
    kc = W.normal_bf16(rng, (B, G, NR, d))
    Q = W.normal_bf16(rng, (B, G, nf, d))
    tau = float(np.sqrt(d))
    got = gpu_head_softmax(Q, kc, T, k, 1, n_local, T - 1, tau, windows,
                           tune={"select_chunk": int(chunk)})
    _hsm_check(got, Q, kc, T, k, 1, n_local, T - 1, tau, windows, "head softmax")


@pytest.mark.parametrize("windows", [False, True])
def test_head_softmax_query_inside_the_sequence_and_default_tau(windows):
    """A query before the end (q_start < T - 1) normalises over the rows it
    sees only; tau <= 0 means sqrt(d)."""
    rng = W.rng_for(150, int(windows))
    B, G, nf, d, T = 2, 2, 4, 128, 12000
    NR = oracle.window_count(T) if windows else (T + 63) // 64
    kc = W.normal_bf16(rng, (B, G, NR, d))
    Q = W.normal_bf16(rng, (B, G, nf, d))
    q = 7000 + 21
    got = gpu_head_softmax(Q, kc, T, 12, 1, 2, q, 0.0, windows)
    _hsm_check(got, Q, kc, T, 12, 1, 2, q, float(np.sqrt(d)), windows, "inside")


@pytest.mark.parametrize("binned", [False, True])
@pytest.mark.parametrize("chunk", ["0", "256"])
@pytest.mark.parametrize("windows", [False, True])
def test_head_softmax_exact_ties_lower_index_wins(windows, chunk, binned):
    """Key rows drawn from six distinct rows with integer entries along the
    heads' axes: every product is exact, equal rows weigh exactly the same
    on both sides, and the lower block index must win every tie."""
    tune = {"select_chunk": int(chunk), "select_binned": int(binned)}
    rng = np.random.default_rng(151)
    B, G, nf, d, T = 2, 2, 4, 128, 1500 * 64
    NR = oracle.window_count(T) if windows else T // 64
    base = np.zeros((6, d), np.float32)
    base[:, :nf] = rng.integers(-2, 3, (6, nf))
    kc = W.f32_to_bf16_bits(base[rng.integers(0, 6, (B, G, NR))])
    Qf = np.zeros((B, G, nf, d), np.float32)
    for h in range(nf):
        Qf[:, :, h, h] = 1.0
    Q = W.f32_to_bf16_bits(Qf)
    for k in (1, 17, 64, 100):
        got = gpu_head_softmax(Q, kc, T, k, 1, 2, T - 1, 1.0, windows, tune=tune)
        ora = oracle.select_head_softmax(Q, kc, T, k, 1, 2, T - 1, 1.0, windows=windows)[0]
        assert np.array_equal(got, ora), "k=%d" % k


@pytest.mark.parametrize("k,n_init,n_local", [(0, 1, 2), (61, 1, 2), (70, 1, 2), (5, 0, 0),
                                              (5, 3, 7), (1, 0, 1)])
@pytest.mark.parametrize("windows", [False, True])
def test_head_softmax_degenerate_budgets(k, n_init, n_local, windows):
    rng = W.rng_for(152, k * 100 + n_init * 10 + n_local + 1000 * int(windows))
    B, G, nf, T = 2, 2, 4, 64 * 64
    NR = oracle.window_count(T) if windows else T // 64
    kc = W.normal_bf16(rng, (B, G, NR, 128))
    Q = W.normal_bf16(rng, (B, G, nf, 128))
    got = gpu_head_softmax(Q, kc, T, k, n_init, n_local, T - 1, 11.3, windows)
    _hsm_check(got, Q, kc, T, k, n_init, n_local, T - 1, 11.3, windows, "degenerate")


@pytest.mark.parametrize("chunk", ["0", "256"])
@pytest.mark.parametrize("windows", [False, True])
def test_head_softmax_per_sequence_lengths(windows, chunk):
    """Sequences of different lengths in one batch, one invalid: each set is
    the oracle's on that sequence alone; the invalid one is all -1.  A second
    call on the same workspace gives the same sets (tickets back at zero)."""
    tune = {"select_chunk": int(chunk)}
    rng = W.rng_for(153, int(windows))
    B, G, nf, d, T, k = 5, 2, 4, 128, 20000, 16
    lens = [T, 3000 + 17, 70, 0, 9000]
    NR = oracle.window_count(T) if windows else (T + 63) // 64
    kc = W.normal_bf16(rng, (B, G, NR, d))
    Q = W.normal_bf16(rng, (B, G, nf, d))
    tau = 11.0
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = abi.make_params(B, G * nf, G, T, k, seq_len=sl, tune=tune)
    op = abi.SPARDA_OP_HEAD_SOFTMAX_WINDOWS if windows else abi.SPARDA_OP_HEAD_SOFTMAX
    ws = abi.workspace(op, p, 1, nf)
    got = gpu_head_softmax(Q, kc, T, k, 1, 2, T - 1, tau, windows, lens=lens, ws=ws, tune=tune)
    again = gpu_head_softmax(Q, kc, T, k, 1, 2, T - 1, tau, windows, lens=lens, ws=ws, tune=tune)
    assert np.array_equal(got, again)
    for b, L in enumerate(lens):
        if L == 0:
            assert np.all(got[b] == -1)
            continue
        nr = oracle.window_count(L) if windows else (L + 63) // 64
        Qb = np.ascontiguousarray(Q[b:b + 1])
        kb = np.ascontiguousarray(kc[b:b + 1, :, :nr])
        _hsm_check(got[b:b + 1], Qb, kb, L, k, 1, 2, L - 1, tau, windows, "len %d" % L)


def test_head_softmax_rejects_bad_arguments():
    B, G, nf, T = 1, 2, 4, 4096
    p = abi.make_params(B, G * nf, G, T, 8)
    kc = torch.zeros(B, G, T // 64, 128, dtype=torch.bfloat16, device="cuda")
    Q = torch.zeros(B, G, nf, 128, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(B, G, 11, dtype=torch.int32, device="cuda")
    ws = abi.workspace(abi.SPARDA_OP_HEAD_SOFTMAX, p, 1, nf)
    for args, status in [((nf, T, 1.0), abi.SPARDA_EINVAL),        # query past the end
                         ((0, T - 1, 1.0), abi.SPARDA_EINVAL),     # no heads
                         ((32, T - 1, 1.0), abi.SPARDA_EUNSUPPORTED),
                         ((nf, T - 1, float("nan")), abi.SPARDA_EINVAL)]:
        with pytest.raises(abi.SpardaError) as e:
            abi.sparda_head_softmax_select(p, Q, args[0], args[1], args[2], kc, idx, ws)
        assert e.value.status == status
    with pytest.raises(abi.SpardaError) as e:
        abi.sparda_head_softmax_select(p, Q, nf, T - 1, 1.0, kc, idx, None)
    assert e.value.status == abi.SPARDA_EWORKSPACE
    assert abi.sparda_workspace_size(abi.SPARDA_OP_HEAD_SOFTMAX, p, 2, nf) == 0   # decode only


# --------------------------------------------------------------------------
# per-sequence lengths (decode) and a real model's budget
# --------------------------------------------------------------------------

def test_varlen_compress_leaves_blocks_past_the_end():
    rng = W.rng_for(100)
    B, G, T, d = 3, 2, 4096 + 5, 128
    lens = [1000, 64, T]
    K = W.normal_bf16(rng, (B, G, T, d))
    NB = (T + 63) // 64
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = abi.make_params(B, G, G, T, 1, seq_len=sl)
    kc32 = torch.full((B, G, NB, d), 7.0, dtype=torch.float32, device="cuda")
    abi.sparda_compress_keys(p, dev_bf16(K), T * d, d, kc32, None)
    torch.cuda.synchronize()
    got = kc32.cpu().numpy()
    for b, L in enumerate(lens):
        o64, _ = oracle.compress_keys(np.ascontiguousarray(K[b:b + 1, :, :L]))
        nb = (L + 63) // 64
        assert np.abs(got[b, :, :nb] - o64[0]).max() <= 1e-3
        assert np.all(got[b, :, nb:] == 7.0)


@pytest.mark.parametrize("chunk", ["0", "256"])
def test_varlen_decode_select_and_attention(chunk):
    """Four sequences of different lengths in one batch: each one's set and
    attention output equal the oracle run on that sequence alone."""
    rng = W.rng_for(101)
    B, G, R, T, d, k = 4, 2, 4, 20000, 128, 16
    lens = [T, 3000 + 17, 70, 9000]
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    Q = W.normal_bf16(rng, (B, G * R, d))
    F = W.normal_bf16(rng, (B, 1, G, 1, d))
    NB = (T + 63) // 64
    S = k + 3
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = abi.make_params(B, G * R, G, T, k, seq_len=sl, tune={"select_chunk": int(chunk)})
    Kd, Vd = dev_bf16(K), dev_bf16(V)
    kc = torch.zeros(B, G, NB, d, dtype=torch.bfloat16, device="cuda")
    abi.sparda_compress_keys(p, Kd, T * d, d, None, kc)
    idx = torch.full((B, 1, G, S), -7, dtype=torch.int32, device="cuda")
    abi.sparda_forecast_select(p, dev_bf16(F), 1, 1, T - 1, kc, idx,
                               abi.workspace(abi.SPARDA_OP_SELECT, p, 1, 1))
    O = torch.empty(B, G * R, d, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.sparda_sparse_attn_decode(p, dev_bf16(Q), Kd, Vd, T * d, 64 * d, idx.view(B, G, S), 0, O,
                                  abi.workspace(abi.SPARDA_OP_ATTN_DECODE, p), status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kcb = host_bits(kc)
    got_idx = idx.cpu().numpy()
    got_o = host_bits(O)
    for b, L in enumerate(lens):
        Fb = F[b:b + 1]
        kcl = np.ascontiguousarray(kcb[b:b + 1, :, :(L + 63) // 64])
        ora, kth, kth1 = oracle.select(Fb, kcl, k, 1, 2, L - 1)
        check_sets(got_idx[b:b + 1], ora, kth, kth1, scores_f64(Fb, kcl), "varlen b=%d" % b,
                   q_pos=L - 1, n_init=1, n_local=2)
        o = oracle.sparse_attention(Q[b:b + 1].reshape(1, 1, G * R, d),
                                    np.ascontiguousarray(K[b:b + 1, :, :L]),
                                    np.ascontiguousarray(V[b:b + 1, :, :L]),
                                    got_idx[b:b + 1], L - 1, L)
        check_attention(got_o[b:b + 1].reshape(1, 1, G * R, d), o, "varlen attention b=%d" % b)


def test_varlen_invalid_length_gives_empty_outputs():
    B, G, T, d, k = 2, 1, 4096, 128, 4
    sl = torch.tensor([T, 0], dtype=torch.int32, device="cuda")
    p = abi.make_params(B, 4, G, T, k, seq_len=sl)
    rng = W.rng_for(102)
    kc = dev_bf16(W.normal_bf16(rng, (B, G, T // 64, d)))
    F = dev_bf16(W.normal_bf16(rng, (B, 1, G, 1, d)))
    idx = torch.full((B, 1, G, k + 3), -7, dtype=torch.int32, device="cuda")
    abi.sparda_forecast_select(p, F, 1, 1, T - 1, kc, idx, abi.workspace(abi.SPARDA_OP_SELECT, p, 1, 1))
    KV = dev_bf16(W.normal_bf16(rng, (B, G, T, d)))
    good = torch.tensor([[[0, 5, 9, 62, 63, -1, -1]]] * B, dtype=torch.int32, device="cuda").view(B, G, 7)
    O = torch.full((B, 4, d), 3.0, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.sparda_sparse_attn_decode(p, dev_bf16(W.normal_bf16(rng, (B, 4, d))), KV, KV, T * d, 64 * d,
                                  good, 0, O, abi.workspace(abi.SPARDA_OP_ATTN_DECODE, p), status)
    torch.cuda.synchronize()
    assert np.all(idx.cpu().numpy()[1] == -1) and not np.any(idx.cpu().numpy()[0] == -7)
    assert abi.sparda_status_from_device(int(status.item())) == abi.SPARDA_ERANGE
    assert torch.all(O[1] == 0) and torch.isfinite(O[0].float()).all()


def test_varlen_prefetch_keeps_each_sequences_resident_blocks():
    rng = W.rng_for(103)
    B, G, NB, d, k = 2, 2, 40, 128, 5
    T = NB * 64
    lens = [T, 1000]
    S = k + 3
    host = W.normal_bf16(rng, (B, G, NB, 2, 64, d))
    idx = np.zeros((B, G, S), np.int32)
    for b, L in enumerate(lens):
        c = (L - 1) // 64
        for g in range(G):
            top = sorted(rng.choice(np.arange(1, c - 1), k, replace=False).tolist())
            idx[b, g] = [0] + top + [c - 1, c]
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = abi.make_params(B, G * 4, G, T, k, seq_len=sl)
    slots = torch.zeros(B, G, S, 2, 64, d, dtype=torch.bfloat16, device="cuda")
    abi.sparda_prefetch_blocks(p, _pinned_bf16(host), torch.from_numpy(idx).cuda(), slots, True)
    torch.cuda.synchronize()
    got = host_bits(slots)
    for b, L in enumerate(lens):
        ora = oracle.gather_blocks(host[b:b + 1], idx[b:b + 1], L - 1, 1, 2, True)
        assert np.array_equal(got[b:b + 1], ora), b


@pytest.mark.parametrize("n_local,chunk", [(2, "0"), (0, "0"), (1, "512")])
def test_varlen_window_grid(n_local, chunk):
    """Window compression and window selection with per-sequence lengths:
    windows not complete inside a sequence are left untouched and never
    scored (with n_local = 0 the query's own partial block is a candidate
    and scores only through the windows its sequence completes)."""
    rng = W.rng_for(105 + n_local)
    B, G, T, d, k = 3, 2, 12000, 128, 12
    lens = [T, 5000 + 45, 1030]
    K = W.normal_bf16(rng, (B, G, T, d))
    F = W.normal_bf16(rng, (B, 1, G, 1, d))
    NW = oracle.window_count(T)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = abi.make_params(B, G, G, T, k, 1, n_local, seq_len=sl, tune={"select_chunk": int(chunk)})
    kw32 = torch.full((B, G, NW, d), 7.0, dtype=torch.float32, device="cuda")
    kw16 = torch.zeros(B, G, NW, d, dtype=torch.bfloat16, device="cuda")
    abi.sparda_compress_windows(p, dev_bf16(K), T * d, d, 32, 16, kw32, kw16)
    S = k + 1 + n_local
    idx = torch.full((B, 1, G, S), -7, dtype=torch.int32, device="cuda")
    abi.sparda_forecast_select_windows(p, dev_bf16(F), 1, 1, T - 1, kw16, 32, 16, idx,
                                       abi.workspace(abi.SPARDA_OP_SELECT_WINDOWS, p, 1, 1))
    torch.cuda.synchronize()
    got32, got16, got_idx = kw32.cpu().numpy(), host_bits(kw16), idx.cpu().numpy()
    for b, L in enumerate(lens):
        nw = oracle.window_count(L)
        o64, o16 = oracle.compress_windows(np.ascontiguousarray(K[b:b + 1, :, :L]))
        check_compressed(got32[b:b + 1, :, :nw], got16[b:b + 1, :, :nw], o64, o16)
        assert np.all(got32[b, :, nw:] == 7.0)
        kwl = np.ascontiguousarray(got16[b:b + 1, :, :nw])
        Fb = F[b:b + 1]
        ora, kth, kth1 = oracle.select_windows(Fb, kwl, L, k, 1, n_local, L - 1)
        check_sets(got_idx[b:b + 1], ora, kth, kth1, pooled_scores_f64(Fb, kwl, (L + 63) // 64),
                   "varlen windows b=%d" % b, q_pos=L - 1, n_init=1, n_local=n_local)


@pytest.mark.parametrize("nq,pool", [(96, 1), (5, 1), (80, 4), (3, 4)])
def test_varlen_prefill_select(nq, pool):
    """A prefill chunk per sequence of different lengths: each sequence's
    chunk is its last nq tokens.  The tensor-core path (nq >= 64) and the
    streaming path, on blocks and on the window grid; one sequence shorter
    than the chunk gets empty sets."""
    rng = W.rng_for(106, nq * 10 + pool)
    B, G, T, d, k = 4, 2, 12000, 128, 10
    lens = [T, 7000 + 13, 200, nq - 1]
    F = W.normal_bf16(rng, (B, nq, G, 1, d))
    NB = (T + 63) // 64
    rows = NB if pool == 1 else oracle.window_count(T)
    kc = W.normal_bf16(rng, (B, G, rows, d))
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = abi.make_params(B, G, G, T, k, seq_len=sl)
    S = k + 3
    idx = torch.full((B, nq, G, S), -7, dtype=torch.int32, device="cuda")
    if pool == 1:
        abi.sparda_forecast_select(p, dev_bf16(F), nq, 1, T - nq, dev_bf16(kc), idx,
                                   abi.workspace(abi.SPARDA_OP_SELECT, p, nq, 1))
    else:
        abi.sparda_forecast_select_windows(p, dev_bf16(F), nq, 1, T - nq, dev_bf16(kc), 32, 16, idx,
                                           abi.workspace(abi.SPARDA_OP_SELECT_WINDOWS, p, nq, 1))
    torch.cuda.synchronize()
    got = idx.cpu().numpy()
    for b, L in enumerate(lens):
        if L < nq:
            assert np.all(got[b] == -1), "invalid length b=%d" % b
            continue
        Fb = F[b:b + 1]
        if pool == 1:
            kb = np.ascontiguousarray(kc[b:b + 1, :, :(L + 63) // 64])
            ora, kth, kth1 = oracle.select(Fb, kb, k, 1, 2, L - nq)
            sc = scores_f64(Fb, kb)
        else:
            kb = np.ascontiguousarray(kc[b:b + 1, :, :oracle.window_count(L)])
            ora, kth, kth1 = oracle.select_windows(Fb, kb, L, k, 1, 2, L - nq)
            sc = pooled_scores_f64(Fb, kb, (L + 63) // 64)
        check_sets(got[b:b + 1], ora, kth, kth1, sc, "varlen prefill b=%d" % b,
                   q_pos=L - nq + np.arange(nq)[None, :], n_init=1, n_local=2)


def test_varlen_prefill_attention():
    """Prefill attention with a chunk per sequence at its own end; a sequence
    shorter than the chunk gets a zero output and the range bit."""
    rng = W.rng_for(107)
    B, G, R, T, d, k, nq = 3, 2, 4, 5000, 128, 8, 70
    lens = [T, 2000 + 31, nq - 5]
    Q = W.normal_bf16(rng, (B, nq, G * R, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    F = W.normal_bf16(rng, (B, nq, G, 1, d))
    S = k + 3
    idx = np.full((B, nq, G, S), -1, np.int32)
    for b, L in enumerate(lens[:2]):
        _, kcb = oracle.compress_keys(np.ascontiguousarray(K[b:b + 1, :, :L]))
        idx[b:b + 1], _, _ = oracle.select(F[b:b + 1], kcb, k, 1, 2, L - nq)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = abi.make_params(B, G * R, G, T, k, seq_len=sl)
    O = torch.full((B, nq, G * R, d), 5.0, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # the short sequence is given a list anyway, so its blocks are flagged
    idx[2] = idx[1]
    abi.sparda_sparse_attn_prefill(p, dev_bf16(Q), nq, T - nq, dev_bf16(K), dev_bf16(V), T * d, d,
                                   torch.from_numpy(idx).cuda(), O,
                                   abi.workspace(abi.SPARDA_OP_ATTN_PREFILL, p, nq), status)
    torch.cuda.synchronize()
    got = host_bits(O)
    for b, L in enumerate(lens[:2]):
        ora = oracle.sparse_attention(Q[b:b + 1], np.ascontiguousarray(K[b:b + 1, :, :L]),
                                      np.ascontiguousarray(V[b:b + 1, :, :L]), idx[b:b + 1], L - nq, L)
        check_attention(got[b:b + 1], ora, "varlen prefill attention b=%d" % b)
    assert torch.all(O[2] == 0)
    assert abi.sparda_status_from_device(int(status.item())) == abi.SPARDA_ERANGE


@pytest.mark.parametrize("k,n_init,n_local", [(63, 1, 32), (24, 1, 16)])
def test_real_model_budget(k, n_init, n_local):
    """A real model's budget: 96 blocks of which 32 (2048 tokens) are the
    local window and one the initial block, leaving 63 to top-k; and a
    16-block local window with 24 query-aware blocks."""
    rng = W.rng_for(104)
    B, G, R, T, d = 2, 2, 4, 16384, 128
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    F = W.normal_bf16(rng, (B, 1, G, 1, d))
    Q = W.normal_bf16(rng, (B, G * R, d))
    _, kcb = oracle.compress_keys(K)
    ora, kth, kth1 = oracle.select(F, kcb, k, n_init, n_local, T - 1)
    got = gpu_select(F, kcb, k, n_init, n_local, T - 1, T, Hq=G * R)
    check_sets(got, ora, kth, kth1, scores_f64(F, kcb), "budget", q_pos=T - 1, n_init=n_init,
               n_local=n_local)
    idx = got[:, 0]
    S = k + n_init + n_local
    assert idx.shape[-1] == S and (idx >= 0).all()
    o = gpu_decode(Q, K, V, idx, T, k, n_init, n_local)
    ora_o = oracle.sparse_attention(Q.reshape(B, 1, G * R, d), K, V, idx.reshape(B, 1, G, S), T - 1, T)
    check_attention(o.reshape(B, 1, G * R, d), ora_o, "budget attention")


# --------------------------------------------------------------------------
# decode attention
# --------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["decode_b1_t4k", "decode_b4_t32k_planted"])
def test_decode_attention_configs(name):
    w = W.WORKLOADS[name]
    x = W.decode_inputs(w)
    _, kcb = oracle.compress_keys(x["K"])
    idx, _, _ = oracle.select(x["F"].reshape(w.B, 1, w.G, 1, w.d), kcb, w.k, w.n_init, w.n_local, w.T - 1)
    Q = x["Q"]
    ora = oracle.sparse_attention(Q.reshape(w.B, 1, w.Hq, w.d), x["K"], x["V"], idx, w.T - 1, w.T)
    got = gpu_decode(Q, x["K"], x["V"], idx[:, 0], w.T, w.k, w.n_init, w.n_local)
    check_attention(got, ora[:, 0], name)


def test_decode_every_block_is_dense_causal():
    w = W.WORKLOADS["decode_b1_t4k"]
    x = W.decode_inputs(w)
    NB = w.NB
    idx = np.broadcast_to(np.arange(NB, dtype=np.int32), (w.B, w.G, NB)).copy()
    got = gpu_decode(x["Q"], x["K"], x["V"], idx, w.T, NB - 3)
    dense = oracle.dense_causal_attention(x["Q"].reshape(w.B, 1, w.Hq, w.d), x["K"], x["V"], w.T - 1)
    check_attention(got, dense[:, 0], "dense")


@pytest.mark.parametrize("R,G", [(1, 4), (2, 4), (4, 2), (8, 2), (16, 1)])
@pytest.mark.parametrize("T", [2048, 2048 + 17])
def test_decode_group_ratios_and_ragged_tail(R, G, T):
    rng = W.rng_for(20, R * 1000 + T)
    B, d, k = 3, 128, 12
    Hq = R * G
    Q = W.normal_bf16(rng, (B, Hq, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    F = W.normal_bf16(rng, (B, 1, G, 1, d))
    _, kcb = oracle.compress_keys(K)
    idx, _, _ = oracle.select(F, kcb, k, 1, 2, T - 1)
    ora = oracle.sparse_attention(Q.reshape(B, 1, Hq, d), K, V, idx, T - 1, T)
    got = gpu_decode(Q, K, V, idx[:, 0], T, k)
    check_attention(got, ora[:, 0], "R=%d T=%d" % (R, T))


def test_decode_padding_entries_are_skipped():
    rng = W.rng_for(21)
    B, G, R, T, d = 2, 2, 4, 640, 128                     # 10 blocks, 7 candidates < k
    k = 12
    Q = W.normal_bf16(rng, (B, G * R, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    F = W.normal_bf16(rng, (B, 1, G, 1, d))
    _, kcb = oracle.compress_keys(K)
    idx, _, _ = oracle.select(F, kcb, k, 1, 2, T - 1)
    assert (idx == -1).any()
    ora = oracle.sparse_attention(Q.reshape(B, 1, G * R, d), K, V, idx, T - 1, T)
    got = gpu_decode(Q, K, V, idx[:, 0], T, k)
    check_attention(got, ora[:, 0], "padding")


def test_decode_slot_mode_on_interleaved_slots():
    rng = W.rng_for(22)
    B, G, R, NB, d, k = 2, 4, 4, 40, 128, 8
    T = NB * 64
    S = k + 3
    Q = W.normal_bf16(rng, (B, G * R, d))
    KV = W.normal_bf16(rng, (B, G, NB, 2, 64, d))         # host layout
    F = W.normal_bf16(rng, (B, 1, G, 1, d))
    K = np.ascontiguousarray(KV[:, :, :, 0].reshape(B, G, T, d))
    V = np.ascontiguousarray(KV[:, :, :, 1].reshape(B, G, T, d))
    _, kcb = oracle.compress_keys(K)
    idx, _, _ = oracle.select(F, kcb, k, 1, 2, T - 1)
    ora = oracle.sparse_attention(Q.reshape(B, 1, G * R, d), K, V, idx, T - 1, T)
    slots = np.ascontiguousarray(KV[np.arange(B)[:, None, None], np.arange(G)[None, :, None], idx[:, 0]])
    got = gpu_decode(Q, slots, None, idx[:, 0], T, k, addr_mode=abi.SPARDA_ADDR_SLOT,
                     bg_stride=S * 2 * 64 * d, blk_stride=2 * 64 * d)
    check_attention(got, ora[:, 0], "slots")
    # the same blocks addressed by id in the full interleaved host layout
    got2 = gpu_decode(Q, KV, None, idx[:, 0], T, k, addr_mode=abi.SPARDA_ADDR_LOGICAL,
                      bg_stride=NB * 2 * 64 * d, blk_stride=2 * 64 * d)
    check_attention(got2, ora[:, 0], "interleaved")


def test_decode_out_of_range_ids_are_flagged_and_skipped():
    rng = W.rng_for(23)
    B, G, R, T, d = 1, 2, 4, 1024, 128
    Q = W.normal_bf16(rng, (B, G * R, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    idx = np.array([[[0, 3, 99, 14, 15], [0, 5, 16, 14, 15]]], np.int32)   # 99 and 16 >= NB
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = gpu_decode(Q, K, V, idx, T, 2, status=status)
    assert abi.sparda_status_from_device(int(status.item())) == abi.SPARDA_ERANGE
    clean = np.where(idx >= 16, -1, idx)
    ora = oracle.sparse_attention(Q.reshape(B, 1, G * R, d), K, V, clean[:, None], T - 1, T)
    check_attention(got, ora[:, 0], "range")


# --------------------------------------------------------------------------
# prefetch
# --------------------------------------------------------------------------

def _pinned_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory()


@pytest.mark.parametrize("skip_resident", [False, True])
def test_prefetch_parity(skip_resident):
    rng = W.rng_for(30)
    B, G, NB, d, k = 3, 4, 50, 128, 9
    T = NB * 64
    S = k + 3
    host = W.normal_bf16(rng, (B, G, NB, 2, 64, d))
    kc = W.normal_bf16(rng, (B, G, NB, d))
    F = W.normal_bf16(rng, (B, 1, G, 1, d))
    idx, _, _ = oracle.select(F, kc, k, 1, 2, T - 1)
    idx = idx[:, 0]
    p = abi.make_params(B, G * 4, G, T, k)
    hkv = _pinned_bf16(host)
    slots = Guarded((B, G, S, 2, 64, d), torch.bfloat16, fill=0)
    abi.sparda_prefetch_blocks(p, hkv, torch.from_numpy(idx).cuda(), slots.t, skip_resident)
    ora = oracle.gather_blocks(host, idx, T - 1, 1, 2, skip_resident)
    assert np.array_equal(host_bits(slots.check("slots")), ora)


def test_prefetch_flags_out_of_range_and_rejects_pageable_memory():
    B, G, NB, d = 1, 2, 8, 128
    host = np.zeros((B, G, NB, 2, 64, d), np.uint16)
    host[0, 1, 3] = 7
    p = abi.make_params(B, 8, G, NB * 64, 2)
    idx = torch.tensor([[[0, 3, 6, 7, 0], [0, 3, 50, 6, 7]]], dtype=torch.int32, device="cuda")[:, :, :5]
    p = abi.make_params(B, 8, G, NB * 64, 2)
    slots = torch.zeros(B, G, 5, 2, 64, d, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.sparda_prefetch_blocks(p, _pinned_bf16(host), idx, slots, False, 0, status)
    torch.cuda.synchronize()
    assert abi.sparda_status_from_device(int(status.item())) == abi.SPARDA_ERANGE
    assert np.array_equal(host_bits(slots)[0, 1, 1], host[0, 1, 3])
    pageable = torch.from_numpy(host.view(np.int16)).view(torch.bfloat16)
    with pytest.raises(abi.SpardaError) as e:
        abi.sparda_prefetch_blocks(p, pageable, idx, slots, False)
    assert e.value.status == abi.SPARDA_EINVAL


# --------------------------------------------------------------------------
# decode append: new K/V rows and the incremental compressed key
# --------------------------------------------------------------------------

@pytest.mark.parametrize("interleaved", [False, True])
def test_append_matches_full_compression(interleaved):
    """Append 150 tokens one at a time after a 100-token prefix: after every
    append the cache holds the new rows and the compressed keys equal a full
    compression of positions 0..pos, bit for bit (fp32 and bf16); at the end
    they also match the oracle."""
    rng = W.rng_for(50 + interleaved)
    B, G, d, T0, T = 2, 3, 128, 100, 250
    NB = (T + 63) // 64
    p = abi.make_params(B, G, G, T, 1)
    newK = W.normal_bf16(rng, (T - T0, B, G, d))
    newV = W.normal_bf16(rng, (T - T0, B, G, d))
    K0 = W.normal_bf16(rng, (B, G, T0, d))
    V0 = W.normal_bf16(rng, (B, G, T0, d))
    if interleaved:  # [B][G][NB][2][64][d]
        cache = torch.zeros(B, G, NB, 2, 64, d, dtype=torch.bfloat16, device="cuda")
        for t in range(T0):
            cache[:, :, t // 64, 0, t % 64] = dev_bf16(K0[:, :, t])
            cache[:, :, t // 64, 1, t % 64] = dev_bf16(V0[:, :, t])
        Kd, Vd = cache, cache.view(-1)[64 * d:]
        bg, blk = NB * 2 * 64 * d, 2 * 64 * d
    else:
        Kd = torch.zeros(B, G, T, d, dtype=torch.bfloat16, device="cuda")
        Vd = torch.zeros(B, G, T, d, dtype=torch.bfloat16, device="cuda")
        Kd[:, :, :T0] = dev_bf16(K0)
        Vd[:, :, :T0] = dev_bf16(V0)
        bg, blk = T * d, 64 * d
    kc32 = torch.zeros(B, G, NB, d, dtype=torch.float32, device="cuda")
    kc16 = torch.zeros(B, G, NB, d, dtype=torch.bfloat16, device="cuda")
    # the prefix: compress positions 0..T0-1
    pp = abi.make_params(B, G, G, T0, 1)
    if interleaved:
        # each block of 64 rows compresses like a short sequence of its own
        for j in range((T0 + 63) // 64):
            n = min(64, T0 - 64 * j)
            pj = abi.make_params(B, G, G, n, 1)
            tmp32 = torch.zeros(B, G, 1, d, dtype=torch.float32, device="cuda")
            tmp16 = torch.zeros(B, G, 1, d, dtype=torch.bfloat16, device="cuda")
            abi.sparda_compress_keys(pj, cache[:, :, j, 0], NB * 2 * 64 * d, d, tmp32, tmp16)
            kc32[:, :, j] = tmp32[:, :, 0]
            kc16[:, :, j] = tmp16[:, :, 0]
    else:
        tmp32 = torch.zeros(B, G, (T0 + 63) // 64, d, dtype=torch.float32, device="cuda")
        tmp16 = torch.zeros(B, G, (T0 + 63) // 64, d, dtype=torch.bfloat16, device="cuda")
        abi.sparda_compress_keys(pp, Kd, bg, d, tmp32, tmp16)
        kc32[:, :, :(T0 + 63) // 64] = tmp32
        kc16[:, :, :(T0 + 63) // 64] = tmp16
    for i, pos in enumerate(range(T0, T)):
        abi.sparda_append_kv(p, pos, dev_bf16(newK[i]), dev_bf16(newV[i]), Kd, Vd, bg, blk, kc32,
                             kc16)
        if pos % 37 == 0 or pos == T - 1 or pos % 64 in (0, 63):
            torch.cuda.synchronize()
            # the full compression of positions 0..pos, from the same cache
            c = pos // 64
            n = pos - 64 * c + 1
            if interleaved:
                pj = abi.make_params(B, G, G, n, 1)
                ref32 = torch.zeros(B, G, 1, d, dtype=torch.float32, device="cuda")
                ref16 = torch.zeros(B, G, 1, d, dtype=torch.bfloat16, device="cuda")
                abi.sparda_compress_keys(pj, cache[:, :, c, 0], NB * 2 * 64 * d, d, ref32, ref16)
                ref32, ref16 = ref32[:, :, 0], ref16[:, :, 0]
            else:
                pf = abi.make_params(B, G, G, pos + 1, 1)
                r32 = torch.zeros(B, G, c + 1, d, dtype=torch.float32, device="cuda")
                r16 = torch.zeros(B, G, c + 1, d, dtype=torch.bfloat16, device="cuda")
                abi.sparda_compress_keys(pf, Kd, bg, d, r32, r16)
                ref32, ref16 = r32[:, :, c], r16[:, :, c]
            assert torch.equal(kc32[:, :, c], ref32), pos
            assert torch.equal(kc16[:, :, c], ref16), pos
    torch.cuda.synchronize()
    # rows landed where they belong, and the keys match the oracle
    Kall = np.concatenate([K0, newK.transpose(1, 2, 0, 3)], axis=2)
    Vall = np.concatenate([V0, newV.transpose(1, 2, 0, 3)], axis=2)
    if interleaved:
        got_k = host_bits(cache[:, :, :, 0]).reshape(B, G, NB * 64, d)[:, :, :T]
        got_v = host_bits(cache[:, :, :, 1]).reshape(B, G, NB * 64, d)[:, :, :T]
    else:
        got_k, got_v = host_bits(Kd), host_bits(Vd)
    assert np.array_equal(got_k, Kall) and np.array_equal(got_v, Vall)
    o64, o16 = oracle.compress_keys(Kall)
    check_compressed(kc32.cpu().numpy(), host_bits(kc16), o64, o16)


@pytest.mark.parametrize("interleaved", [False, True])
def test_append_windows_matches_full_compression(interleaved):
    """The window grid's append: after each token, the window it completes
    (if any) gets its key; at checkpoints the window keys equal a full window
    compression of positions 0..pos (bit for bit in the [T][d] layout, within
    the key tolerance against the oracle in the interleaved one)."""
    rng = W.rng_for(53 + interleaved)
    B, G, d, T0, T = 2, 2, 128, 40, 200
    NB = (T + 63) // 64
    NW = oracle.window_count(T)
    p = abi.make_params(B, G, G, T, 1)
    Kall = W.normal_bf16(rng, (B, G, T, d))
    if interleaved:
        cache = torch.zeros(B, G, NB, 2, 64, d, dtype=torch.bfloat16, device="cuda")
        for t in range(T0):
            cache[:, :, t // 64, 0, t % 64] = dev_bf16(Kall[:, :, t])
        Kd = cache
        bg, blk = NB * 2 * 64 * d, 2 * 64 * d
    else:
        Kd = torch.zeros(B, G, T, d, dtype=torch.bfloat16, device="cuda")
        Kd[:, :, :T0] = dev_bf16(Kall[:, :, :T0])
        bg, blk = T * d, 64 * d
    V = Kd.view(-1)[64 * d:] if interleaved else torch.zeros_like(Kd)
    kw32 = torch.full((B, G, NW, d), 9.0, dtype=torch.float32, device="cuda")
    kw16 = torch.zeros(B, G, NW, d, dtype=torch.bfloat16, device="cuda")
    # the prefix's windows, from the host keys
    o64, o16 = oracle.compress_windows(Kall[:, :, :T0])
    nw0 = o64.shape[2]
    kw32[:, :, :nw0] = torch.from_numpy(o64.astype(np.float32)).cuda()
    kw16[:, :, :nw0] = dev_bf16(o16)
    zero = torch.zeros(B, G, d, dtype=torch.bfloat16, device="cuda")
    kc16 = torch.zeros(B, G, NB, d, dtype=torch.bfloat16, device="cuda")  # the block keys (unchecked here)
    for pos in range(T0, T):
        abi.sparda_append_kv(p, pos, dev_bf16(Kall[:, :, pos]), zero, Kd, V, bg, blk, None, kc16)
        abi.sparda_append_windows(p, pos, Kd, bg, blk, 32, 16, kw32, kw16)
        if not interleaved and (pos % 16 == 15 or pos == T - 1):
            torch.cuda.synchronize()
            nw = oracle.window_count(pos + 1)
            pf = abi.make_params(B, G, G, pos + 1, 1)
            r32 = torch.zeros(B, G, max(nw, 1), d, dtype=torch.float32, device="cuda")
            r16 = torch.zeros(B, G, max(nw, 1), d, dtype=torch.bfloat16, device="cuda")
            abi.sparda_compress_windows(pf, Kd, bg, d, 32, 16, r32, r16)
            torch.cuda.synchronize()
            assert torch.equal(kw32[:, :, nw0:nw], r32[:, :, nw0:nw]), pos
            assert torch.equal(kw16[:, :, nw0:nw], r16[:, :, nw0:nw]), pos
            assert torch.all(kw32[:, :, nw:] == 9.0), pos  # windows not complete yet stay as they were
    torch.cuda.synchronize()
    o64, o16 = oracle.compress_windows(Kall)
    check_compressed(kw32.cpu().numpy(), host_bits(kw16), o64, o16)


def test_append_windows_per_sequence_positions():
    rng = W.rng_for(55)
    B, G, d, T = 3, 2, 128, 300
    lens = [240, 127, 0]   # position 239 ends window 13; position 126 ends none
    NW = oracle.window_count(T)
    K = W.normal_bf16(rng, (B, G, T, d))
    Kd = dev_bf16(K)
    kw32 = torch.full((B, G, NW, d), 9.0, dtype=torch.float32, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = abi.make_params(B, G, G, T, 1, seq_len=sl)
    abi.sparda_append_windows(p, 0, Kd, T * d, 64 * d, 32, 16, kw32, None)
    torch.cuda.synchronize()
    got = kw32.cpu().numpy()
    w = (239 - 31) // 16
    o64, _ = oracle.compress_windows(np.ascontiguousarray(K[0:1, :, :240]))
    assert np.abs(got[0, :, w] - o64[0, :, w]).max() <= 1e-3
    got[0, :, w] = 9.0
    assert np.all(got == 9.0)  # nothing else was written


def test_append_per_sequence_positions():
    """With per-sequence lengths each sequence appends its new token at its
    own last position (seq_len[b] - 1); the rows land there, and the block's
    compressed key equals a full compression of that sequence, bit for bit.
    A sequence with an invalid length is left untouched."""
    rng = W.rng_for(52)
    B, G, d, T = 4, 2, 128, 300
    lens = [250, 130, 64, 0]
    NB = (T + 63) // 64
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    newK = W.normal_bf16(rng, (B, G, d))
    newV = W.normal_bf16(rng, (B, G, d))
    Kd, Vd = dev_bf16(K), dev_bf16(V)
    kc32 = torch.full((B, G, NB, d), 9.0, dtype=torch.float32, device="cuda")
    kc16 = torch.zeros(B, G, NB, d, dtype=torch.bfloat16, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = abi.make_params(B, G, G, T, 1, seq_len=sl)
    abi.sparda_append_kv(p, 0, dev_bf16(newK), dev_bf16(newV), Kd, Vd, T * d, 64 * d, kc32, kc16)
    # the reference: the same caches with the rows written on the host,
    # compressed in full up to each sequence's length
    Kr, Vr = K.copy(), V.copy()
    for b, L in enumerate(lens):
        if L >= 1:
            Kr[b, :, L - 1] = newK[b]
            Vr[b, :, L - 1] = newV[b]
    r32 = torch.zeros(B, G, NB, d, dtype=torch.float32, device="cuda")
    r16 = torch.zeros(B, G, NB, d, dtype=torch.bfloat16, device="cuda")
    abi.sparda_compress_keys(p, dev_bf16(Kr), T * d, d, r32, r16)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(Kd), Kr) and np.array_equal(host_bits(Vd), Vr)
    got32, got16, ref32, ref16 = kc32.cpu(), kc16.cpu(), r32.cpu(), r16.cpu()
    for b, L in enumerate(lens):
        if L < 1:
            assert torch.all(got32[b] == 9.0)
            continue
        c = (L - 1) // 64
        assert torch.equal(got32[b, :, c], ref32[b, :, c]) and torch.equal(got16[b, :, c], ref16[b, :, c])
        o64, _ = oracle.compress_keys(np.ascontiguousarray(Kr[b:b + 1, :, :L]))
        assert np.abs(got32[b, :, c].numpy() - o64[0, :, c]).max() <= 1e-3
        others = [j for j in range(NB) if j != c]
        assert torch.all(got32[b, :, others] == 9.0)  # only the token's block is written


# --------------------------------------------------------------------------
# device slot cache across decode steps
# --------------------------------------------------------------------------

def _drifting_sets(rng, B, G, S, NB, steps, change):
    """Per step, sorted distinct block sets that keep all but `change` blocks
    of the previous step (plus -1 padding in one row and a stale id)."""
    cur = np.stack([np.stack([rng.choice(NB, S, replace=False) for _ in range(G)]) for _ in range(B)])
    out = []
    for _ in range(steps):
        for b in range(B):
            for g in range(G):
                for s in rng.choice(S, change, replace=False):
                    fresh = np.setdiff1d(np.arange(NB), cur[b, g])
                    cur[b, g, s] = rng.choice(fresh)
        out.append(np.sort(cur, axis=2).astype(np.int32))
    return out


def test_cache_plan_matches_oracle_over_steps():
    rng = np.random.default_rng(40)
    B, G, k, C, NB = 2, 3, 7, 16, 64
    S = k + 3
    p = abi.make_params(B, G, G, NB * 64, k)
    block_of = torch.full((B, G, C), -1, dtype=torch.int32, device="cuda")
    hand = torch.zeros(B, G, dtype=torch.int32, device="cuda")
    phys = torch.empty(B, G, S, dtype=torch.int32, device="cuda")
    fetch = torch.empty_like(phys)
    o_blk = np.full((B, G, C), -1, np.int32)
    o_hand = np.zeros((B, G), np.int32)
    for step, idx in enumerate(_drifting_sets(rng, B, G, S, NB, 25, 3)):
        if step == 4:
            idx[1, 2, -2:] = -1          # a short list
        didx = torch.from_numpy(idx).cuda()
        abi.sparda_cache_plan(p, C, didx, block_of, hand, phys, fetch)
        torch.cuda.synchronize()
        o_phys, o_fetch, o_blk, o_hand = oracle.cache_plan(idx, o_blk, o_hand, NB)
        assert np.array_equal(phys.cpu().numpy(), o_phys), step
        assert np.array_equal(fetch.cpu().numpy(), o_fetch), step
        assert np.array_equal(block_of.cpu().numpy(), o_blk), step
        assert np.array_equal(hand.cpu().numpy(), o_hand), step


def test_cache_plan_rejects_too_few_slots_and_flags_bad_ids():
    p = abi.make_params(1, 1, 1, 64 * 10, 4)        # S = 7
    idx = torch.tensor([[[0, 1, 2, 3, 99, 8, 9]]], dtype=torch.int32, device="cuda")
    blk = torch.full((1, 1, 8), -1, dtype=torch.int32, device="cuda")
    hand = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    phys = torch.empty(1, 1, 7, dtype=torch.int32, device="cuda")
    fetch = torch.empty_like(phys)
    with pytest.raises(abi.SpardaError) as e:
        abi.sparda_cache_plan(p, 6, idx, blk, hand, phys, fetch)
    assert e.value.status == abi.SPARDA_EINVAL
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.sparda_cache_plan(p, 8, idx, blk, hand, phys, fetch, status)
    torch.cuda.synchronize()
    assert abi.sparda_status_from_device(int(status.item())) == abi.SPARDA_ERANGE
    assert phys.cpu().numpy()[0, 0, 4] == -1 and fetch.cpu().numpy()[0, 0, 4] == 0


@pytest.mark.parametrize("R", [4, 8])
def test_cached_prefetch_and_attention_over_steps(R):
    """Plan, fetch only the misses, attend from the cache -- three steps of
    drifting sets: the cache holds the host bytes at every slot a list uses,
    and attention equals the oracle over the logical block ids."""
    rng = np.random.default_rng(41 + R)
    B, G, NB, d, k, C = 2, 2, 96, 128, 13, 24
    T = NB * 64 - 5
    S = k + 3
    host = W.normal_bf16(rng, (B, G, NB, 2, 64, d))
    kc = W.normal_bf16(rng, (B, G, NB, d))
    p = abi.make_params(B, G * R, G, T, k)
    hkv = _pinned_bf16(host)
    gcache = Guarded((B, G, C, 2, 64, d), torch.bfloat16, fill=0)
    gblock_of = Guarded((B, G, C), torch.int32, fill=-1)
    ghand = Guarded((B, G), torch.int32, fill=0)
    gphys = Guarded((B, G, S), torch.int32, fill=0)
    gfetch = Guarded((B, G, S), torch.int32, fill=0)
    cache, block_of, hand, phys, fetch = gcache.t, gblock_of.t, ghand.t, gphys.t, gfetch.t
    gws = guarded_workspace(abi.SPARDA_OP_ATTN_DECODE, p)
    ws = gws.t
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o_cache = np.zeros((B, G, C, 2, 64, d), np.uint16)
    o_blk, o_hand = np.full((B, G, C), -1, np.int32), np.zeros((B, G), np.int32)
    Fb = W.normal_bf16(rng, (B, 1, G, 1, d))
    for step in range(3):
        if step > 0:  # the Forecast drifts a little each step, so most of the set stays
            drift = 0.3 * rng.standard_normal(Fb.shape).astype(np.float32)
            Fb = W.f32_to_bf16_bits(W.bf16_bits_to_f32(Fb) + drift)
        idx, _, _ = oracle.select(Fb, kc, k, 1, 2, T - 1)
        idx = np.ascontiguousarray(idx[:, 0])
        didx = torch.from_numpy(idx).cuda()
        abi.sparda_cache_plan(p, C, didx, block_of, hand, phys, fetch, status)
        abi.sparda_prefetch_cached(p, C, hkv, didx, phys, fetch, cache, 0, status)
        Q = W.normal_bf16(rng, (B, G * R, d))
        gO = Guarded((B, G * R, d), torch.bfloat16)
        O = gO.t
        abi.sparda_sparse_attn_decode_cached(p, C, dev_bf16(Q), cache, didx, phys, O, ws, status)
        for gb, what in ((gcache, "cache"), (gblock_of, "block_of"), (ghand, "hand"),
                         (gphys, "phys"), (gfetch, "fetch"), (gws, "workspace"), (gO, "O")):
            gb.check(what)
        assert int(status.item()) == 0
        o_phys, o_fetch, o_blk, o_hand = oracle.cache_plan(idx, o_blk, o_hand, NB)
        assert np.array_equal(phys.cpu().numpy(), o_phys)
        assert np.array_equal(fetch.cpu().numpy(), o_fetch)
        o_cache = oracle.gather_cached(host, idx, o_phys, o_fetch, o_cache)
        got = host_bits(cache)
        for b in range(B):
            for g in range(G):
                for s in range(S):
                    assert np.array_equal(got[b, g, o_phys[b, g, s]], host[b, g, idx[b, g, s]])
        assert np.array_equal(got, o_cache)
        flat = host.reshape(-1)
        ora = oracle.sparse_attention(Q.reshape(B, 1, G * R, d), flat, flat[64 * d:],
                                      idx.reshape(B, 1, G, S), T - 1, T, 64,
                                      bg_stride=NB * 2 * 64 * d, blk_stride=2 * 64 * d, G=G)
        check_attention(host_bits(O).reshape(B, 1, G * R, d), ora, "cached step %d" % step)


def test_cached_attention_with_lengths():
    """The slot cache's attention (entries read from their slots) with
    per-sequence lengths: each sequence against the oracle over its own
    length, with its lists selected at its own last token."""
    rng = np.random.default_rng(47)
    B, G, R, NB, d, k, C = 2, 2, 4, 80, 128, 11, 20
    T = NB * 64
    lens = [T - 3, 2600 + 17]
    S = k + 3
    host = W.normal_bf16(rng, (B, G, NB, 2, 64, d))
    kc = W.normal_bf16(rng, (B, G, NB, d))
    F = W.normal_bf16(rng, (B, 1, G, 1, d))
    idx = np.empty((B, G, S), np.int32)
    for b, L in enumerate(lens):
        o, _, _ = oracle.select(F[b:b + 1], np.ascontiguousarray(kc[b:b + 1, :, :(L + 63) // 64]),
                                k, 1, 2, L - 1)
        idx[b] = o[0, 0]
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    p = abi.make_params(B, G * R, G, T, k, seq_len=sl)
    cache = torch.zeros(B, G, C, 2, 64, d, dtype=torch.bfloat16, device="cuda")
    block_of = torch.full((B, G, C), -1, dtype=torch.int32, device="cuda")
    hand = torch.zeros(B, G, dtype=torch.int32, device="cuda")
    phys = torch.empty(B, G, S, dtype=torch.int32, device="cuda")
    fetch = torch.empty_like(phys)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    didx = torch.from_numpy(idx).cuda()
    abi.sparda_cache_plan(p, C, didx, block_of, hand, phys, fetch, status)
    abi.sparda_prefetch_cached(p, C, _pinned_bf16(host), didx, phys, fetch, cache, 0, status)
    Q = W.normal_bf16(rng, (B, G * R, d))
    O = torch.empty(B, G * R, d, dtype=torch.bfloat16, device="cuda")
    abi.sparda_sparse_attn_decode_cached(p, C, dev_bf16(Q), cache, didx, phys, O,
                                         abi.workspace(abi.SPARDA_OP_ATTN_DECODE, p), status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = host_bits(O)
    for b, L in enumerate(lens):
        flat = np.ascontiguousarray(host[b:b + 1]).reshape(-1)
        ora = oracle.sparse_attention(Q[b:b + 1].reshape(1, 1, G * R, d), flat, flat[64 * d:],
                                      idx[b:b + 1].reshape(1, 1, G, S), L - 1, L, 64,
                                      bg_stride=NB * 2 * 64 * d, blk_stride=2 * 64 * d, G=G)
        check_attention(got[b:b + 1].reshape(1, 1, G * R, d), ora, "cached with lengths b=%d" % b)


def _t(g):
    return None if g is None else g.t


@pytest.mark.parametrize("case", ["multi_chunk", "one_chunk", "lengths", "big_budget"])
def test_select_cached_matches_oracle_over_steps(case):
    """The cached selection -- selection, slot plan and fetch of the misses
    from one launch -- over five steps of drifting Forecast vectors: the sets
    equal the oracle's selection, and the slot map, fetch flags, cache state
    and slot bytes equal the oracle's plan and gather of those sets; the
    three separate calls on the same inputs leave the same bytes.  Cases: a
    problem in several chunks (the ranking block plans), one chunk per
    problem, and per-sequence lengths with a sequence whose candidates all
    fit the budget, one whose length is invalid (empty set, flagged) and one
    whose set is shorter than the list (-1 padding), and a
    budget of 300 blocks (lists and slot maps longer than the 256 threads of
    a block, the binned threshold search) with 340 slots."""
    seed = {"multi_chunk": 50, "one_chunk": 51, "lengths": 52, "big_budget": 53}[case]
    rng = np.random.default_rng(seed)
    B, G, d, k = (4 if case == "lengths" else 2), 3, 128, 12
    NB = 300 if case == "one_chunk" else 700
    if case == "big_budget":
        G, k, NB = 2, 300, 1500
    T = NB * 64 - 9
    S = k + 3
    C = S + (37 if case == "big_budget" else 5)  # few spare slots: misses recycle slots
    host = W.normal_bf16(rng, (B, G, NB, 2, 64, d))
    kc = W.normal_bf16(rng, (B, G, NB, d))
    lens = [T] * B
    sl = None
    if case == "lengths":
        lens = [T - 3, 64 * 14 + 5, 0, 64 * 5 + 7]  # long; every candidate kept; invalid; padded
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    tune = {"select_chunk": {"multi_chunk": 256, "big_budget": 512}.get(case, 1024)}
    p = abi.make_params(B, G * 4, G, T, k, seq_len=sl, tune=tune)
    hkv = _pinned_bf16(host)
    dkc = dev_bf16(kc)
    st = {}
    for side in ("fused", "split"):
        st[side] = dict(
            idx=Guarded((B, G, S), torch.int32, fill=0),
            cache=Guarded((B, G, C, 2, 64, d), torch.bfloat16, fill=0),
            block_of=Guarded((B, G, C), torch.int32, fill=-1),
            hand=Guarded((B, G), torch.int32, fill=0),
            phys=Guarded((B, G, S), torch.int32, fill=0),
            fetch=Guarded((B, G, S), torch.int32, fill=0),
            ws=guarded_workspace(abi.SPARDA_OP_SELECT, p, 1, 1),
            status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    o_cache = np.zeros((B, G, C, 2, 64, d), np.uint16)
    o_blk, o_hand = np.full((B, G, C), -1, np.int32), np.zeros((B, G), np.int32)
    Fb = W.normal_bf16(rng, (B, 1, G, 1, d))
    fetched = 0
    for step in range(5):
        if step > 0:
            drift = 0.3 * rng.standard_normal(Fb.shape).astype(np.float32)
            Fb = W.f32_to_bf16_bits(W.bf16_bits_to_f32(Fb) + drift)
        dF = dev_bf16(Fb)
        f, s_ = st["fused"], st["split"]
        abi.sparda_forecast_select_cached(p, dF, 1, T - 1, dkc, f["idx"].t, _t(f["ws"]), C,
                                          f["block_of"].t, f["hand"].t, f["phys"].t,
                                          f["fetch"].t, hkv, f["cache"].t, f["status"])
        abi.sparda_forecast_select(p, dF, 1, 1, T - 1, dkc, s_["idx"].t, _t(s_["ws"]),
                                   s_["status"])
        abi.sparda_cache_plan(p, C, s_["idx"].t, s_["block_of"].t, s_["hand"].t, s_["phys"].t,
                              s_["fetch"].t, s_["status"])
        abi.sparda_prefetch_cached(p, C, hkv, s_["idx"].t, s_["phys"].t, s_["fetch"].t,
                                   s_["cache"].t, 0, s_["status"])
        torch.cuda.synchronize()
        for side in st.values():
            for name in ("idx", "cache", "block_of", "hand", "phys", "fetch", "ws"):
                if side[name] is not None:
                    side[name].check("%s step %d" % (name, step))
        want_status = abi.SPARDA_ERANGE if case == "lengths" else abi.SPARDA_OK
        for side in st.values():
            assert abi.sparda_status_from_device(int(side["status"].item())) == want_status
        # the oracle: every sequence's set at its own last token, then the plan
        o_idx = np.full((B, G, S), -1, np.int32)
        for b, L in enumerate(lens):
            if L < 1:
                continue
            o, _, _ = oracle.select(Fb[b:b + 1], np.ascontiguousarray(kc[b:b + 1, :, :(L + 63) // 64]),
                                    k, 1, 2, L - 1)
            o_idx[b] = o[0, 0]
        got_idx = f["idx"].t.cpu().numpy()
        assert np.array_equal(got_idx, o_idx), "sets, step %d" % step
        o_phys, o_fetch, o_blk, o_hand = oracle.cache_plan(o_idx, o_blk, o_hand, NB)
        o_cache = oracle.gather_cached(host, o_idx, o_phys, o_fetch, o_cache)
        assert np.array_equal(f["phys"].t.cpu().numpy(), o_phys), step
        assert np.array_equal(f["fetch"].t.cpu().numpy(), o_fetch), step
        assert np.array_equal(f["block_of"].t.cpu().numpy(), o_blk), step
        assert np.array_equal(f["hand"].t.cpu().numpy(), o_hand), step
        assert np.array_equal(host_bits(f["cache"].t), o_cache), step
        for name in ("idx", "block_of", "hand", "phys", "fetch"):
            assert torch.equal(f[name].t, s_[name].t), (name, step)
        assert torch.equal(f["cache"].t.view(torch.int16), s_["cache"].t.view(torch.int16)), step
        fetched += int(o_fetch.sum())
    # the steps exercise both hits and misses
    assert 0 < fetched < 5 * B * G * S


def test_select_cached_rejects_bad_arguments():
    """Argument checks of the cached selection: fewer slots than list
    entries, and device memory given as the mapped host buffer."""
    B, G, NB, k = 1, 2, 40, 6
    T = NB * 64
    S = k + 3
    p = abi.make_params(B, G * 4, G, T, k)
    dev = torch.device("cuda")
    F = torch.zeros(B, G, 128, dtype=torch.bfloat16, device=dev)
    kc = torch.zeros(B, G, NB, 128, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(B, G, S, dtype=torch.int32, device=dev)
    ws = abi.workspace(abi.SPARDA_OP_SELECT, p, 1, 1)
    blk = torch.full((B, G, S), -1, dtype=torch.int32, device=dev)
    hand = torch.zeros(B, G, dtype=torch.int32, device=dev)
    phys = torch.empty(B, G, S, dtype=torch.int32, device=dev)
    fetch = torch.empty_like(phys)
    cache = torch.empty(B, G, S, 2, 64, 128, dtype=torch.bfloat16, device=dev)
    host = torch.zeros(B, G, NB, 2, 64, 128, dtype=torch.bfloat16).pin_memory()
    for C, hk in ((S - 1, host), (S, cache)):  # too few slots; device memory as the host buffer
        with pytest.raises(abi.SpardaError) as e:
            abi.sparda_forecast_select_cached(p, F, 1, T - 1, kc, idx, ws, C, blk, hand, phys,
                                              fetch, hk, cache)
        assert e.value.status == abi.SPARDA_EINVAL


# --------------------------------------------------------------------------
# prefill attention
# --------------------------------------------------------------------------

@pytest.mark.parametrize("T,nq,R", [(8192, 160, 4), (4096 + 29, 77, 8), (700, 700, 2)])
def test_prefill_attention_parity(T, nq, R):
    rng = W.rng_for(40, T + nq)
    B, G, d, k = 2, 2, 128, 8
    Hq = G * R
    q_start = T - nq
    Q = W.normal_bf16(rng, (B, nq, Hq, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    F = W.normal_bf16(rng, (B, nq, G, 1, d))
    _, kcb = oracle.compress_keys(K)
    idx, _, _ = oracle.select(F, kcb, k, 1, 2, q_start)
    ora = oracle.sparse_attention(Q, K, V, idx, q_start, T)
    p = abi.make_params(B, Hq, G, T, k)
    O = Guarded((B, nq, Hq, d), torch.bfloat16)
    ws = guarded_workspace(abi.SPARDA_OP_ATTN_PREFILL, p, nq)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.sparda_sparse_attn_prefill(p, dev_bf16(Q), nq, q_start, dev_bf16(K), dev_bf16(V), T * d, d,
                                   torch.from_numpy(idx).cuda(), O.t, ws.t, status)
    ws.check("prefill workspace")
    assert int(status.item()) == 0
    check_attention(host_bits(O.check("prefill output")), ora, "prefill T=%d nq=%d" % (T, nq))


@pytest.mark.parametrize("split", ["1", "-1"])
@pytest.mark.parametrize("nq,R", [(1, 4), (1, 16), (96, 4)])
def test_attention_both_slot_protocols(split, nq, R):
    """The per-token attention kernel has two ring protocols: one barrier per
    slot (the default for decode) and K and V tiles refilled separately (its
    default for prefill chunks).  Each is forced on the other workload too
    (prefill through the per-token kernel rather than the block-major one)."""
    tune = {"attn_split_kv": int(split), "attn_prefill_per_token": int(nq > 1)}
    rng = W.rng_for(41, nq * 100 + R)
    B, G, d, k, T = 2, 2, 128, 12, 6000 + 21
    Hq = G * R
    q_start = T - nq
    Q = W.normal_bf16(rng, (B, nq, Hq, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    F = W.normal_bf16(rng, (B, nq, G, 1, d))
    _, kcb = oracle.compress_keys(K)
    idx, _, _ = oracle.select(F, kcb, k, 1, 2, q_start)
    ora = oracle.sparse_attention(Q, K, V, idx, q_start, T)
    if nq == 1:
        got = gpu_decode(Q.reshape(B, Hq, d), K, V, idx[:, 0], T, k, tune=tune)
        check_attention(got.reshape(B, 1, Hq, d), ora, "decode split=%s R=%d" % (split, R))
    else:
        p = abi.make_params(B, Hq, G, T, k, tune=tune)
        O = torch.empty(B, nq, Hq, d, dtype=torch.bfloat16, device="cuda")
        ws = abi.workspace(abi.SPARDA_OP_ATTN_PREFILL, p, nq)
        abi.sparda_sparse_attn_prefill(p, dev_bf16(Q), nq, q_start, dev_bf16(K), dev_bf16(V), T * d,
                                       d, torch.from_numpy(idx).cuda(), O, ws)
        torch.cuda.synchronize()
        check_attention(host_bits(O), ora, "prefill split=%s" % split)


def _prefill_case(B, G, R, T, nq, k, seed, n_init=1, n_local=2):
    rng = W.rng_for(seed, T + nq + R)
    d = 128
    Q = W.normal_bf16(rng, (B, nq, G * R, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    F = W.normal_bf16(rng, (B, nq, G, 1, d))
    _, kcb = oracle.compress_keys(K)
    idx, _, _ = oracle.select(F, kcb, k, n_init, n_local, T - nq)
    return Q, K, V, idx


def _gpu_prefill(Q, K, V, idx, T, k, tune=None, n_init=1, n_local=2, status=None):
    B, nq, Hq, d = Q.shape
    G = K.shape[1]
    p = abi.make_params(B, Hq, G, T, k, n_init, n_local, tune=tune)
    O = Guarded((B, nq, Hq, d), torch.bfloat16, fill=float("nan"))
    ws = guarded_workspace(abi.SPARDA_OP_ATTN_PREFILL, p, nq)
    abi.sparda_sparse_attn_prefill(p, dev_bf16(Q), nq, T - nq, dev_bf16(K), dev_bf16(V), T * d, d,
                                   torch.from_numpy(np.ascontiguousarray(idx)).cuda(), O.t, ws.t,
                                   status)
    ws.check("prefill workspace")
    return host_bits(O.check("prefill output"))


@pytest.mark.parametrize("R,T,nq,k", [(1, 5000 + 13, 300, 12), (16, 3000, 90, 7), (4, 9000, 520, 40),
                                      (2, 640, 640, 3)])
def test_prefill_block_major_matches_oracle_and_per_token_kernel(R, T, nq, k):
    """The block-major prefill kernels (block -> tokens inversion, one read
    of each selected block for all the tokens that chose it, partials merged
    per token) against the oracle and against the per-token kernel, for 1
    and 16 heads per group, chunks whose initial block is chosen by several
    items' worth of tokens, and a chunk that starts at position 0."""
    Q, K, V, idx = _prefill_case(2, 2, R, T, nq, k, 44)
    ora = oracle.sparse_attention(Q, K, V, idx, T - nq, T)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _gpu_prefill(Q, K, V, idx, T, k, status=st)
    assert int(st.item()) == 0
    check_attention(got, ora, "block-major R=%d" % R)
    ref = _gpu_prefill(Q, K, V, idx, T, k, tune={"attn_prefill_per_token": 1})
    check_attention(ref, ora, "per-token R=%d" % R)
    # each is within the tolerance of the oracle, so within twice it of the other
    assert np.abs(bf16_f64(got) - bf16_f64(ref)).max() <= 2e-2


def test_prefill_block_major_skips_and_flags_bad_ids():
    """Ids past a token's own block (or past the sequence) are skipped and
    flagged; the rest of the set is attended as if they were absent."""
    B, G, R, T, nq, k = 1, 2, 4, 4096, 100, 6
    Q, K, V, idx = _prefill_case(B, G, R, T, nq, k, 45)
    bad = idx.copy()
    bad[0, 10, 1, 2] = 9999           # past the sequence
    bad[0, 20, 0, 3] = (T - nq + 20) // 64 + 1   # after the token's own block
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _gpu_prefill(Q, K, V, bad, T, k, status=st)
    assert abi.sparda_status_from_device(int(st.item())) == abi.SPARDA_ERANGE
    clean = bad.copy()
    clean[0, 10, 1, 2] = -1
    clean[0, 20, 0, 3] = -1
    ora = oracle.sparse_attention(Q, K, V, clean, T - nq, T)
    check_attention(got, ora, "bad ids skipped")
