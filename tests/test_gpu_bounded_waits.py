"""The attention kernel's bounded waits, made to run out on purpose.

Every wait of the attention pipeline (a TMA copy landing, a tensor-core
product completing, a ring slot freeing) gives up after
sparda_tuning.attn_wait_cycles SM cycles (about one second by default).
These tests set the bound to one cycle, so waits give up almost at once
while every copy and product already issued still completes.  The call must
then return with SPARDA_DEV_TIMEOUT in the status word after draining what
it issued and freeing its tensor memory, and it must hand in its tickets, so
the next normal call on the same workspace is correct (checked against the
oracle) and the device stays usable.  No wait is left unbounded, no trap is
raised: the device is never faulted.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_sparda_b200 import abi, build
from block_sparse_long_sparda_b200 import workloads as W
from tests.parity import Guarded, check_attention, dev_bf16, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    abi.lib()
    torch.cuda.init()


def _case():
    w = W.WORKLOADS["decode_b4_t32k_planted"]
    x = W.decode_inputs(w)
    _, kcb = oracle.compress_keys(x["K"])
    idx, _, _ = oracle.select(x["F"].reshape(w.B, 1, w.G, 1, w.d), kcb, w.k, w.n_init,
                              w.n_local, w.T - 1)
    ora = oracle.sparse_attention(x["Q"].reshape(w.B, 1, w.Hq, w.d), x["K"], x["V"], idx,
                                  w.T - 1, w.T)
    return w, x, idx[:, 0], ora


@pytest.mark.parametrize("split", [-1, 1])
def test_decode_waits_run_out_then_the_workspace_serves_the_next_call(split):
    w, x, idx, ora = _case()
    p = abi.make_params(w.B, w.Hq, w.G, w.T, w.k, w.n_init, w.n_local,
                        tune={"attn_split_kv": split})
    p_short = abi.make_params(w.B, w.Hq, w.G, w.T, w.k, w.n_init, w.n_local,
                              tune={"attn_split_kv": split, "attn_wait_cycles": 1})
    assert abi.sparda_workspace_size(abi.SPARDA_OP_ATTN_DECODE, p) == \
        abi.sparda_workspace_size(abi.SPARDA_OP_ATTN_DECODE, p_short)
    Q, K, V = dev_bf16(x["Q"]), dev_bf16(x["K"]), dev_bf16(x["V"])
    didx = torch.from_numpy(np.ascontiguousarray(idx)).cuda()
    bg, blk = w.T * w.d, 64 * w.d
    ws = Guarded((abi.sparda_workspace_size(abi.SPARDA_OP_ATTN_DECODE, p),), torch.uint8, fill=0)
    timeouts = 0
    for _ in range(3):
        O = torch.empty(w.B, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        abi.sparda_sparse_attn_decode(p_short, Q, K, V, bg, blk, didx, abi.SPARDA_ADDR_LOGICAL, O,
                                      ws.t, st)
        torch.cuda.synchronize()                     # the call ends: no hang
        word = int(st.item())
        assert word & ~abi.SPARDA_DEV_TIMEOUT == 0, word
        timeouts += word == abi.SPARDA_DEV_TIMEOUT
    assert timeouts > 0, "a one-cycle bound never ran out"
    assert abi.sparda_status_from_device(abi.SPARDA_DEV_TIMEOUT) == abi.SPARDA_ETIMEOUT
    ws.check("workspace after timeouts")
    # the next call relies on every ticket being back at zero: same
    # workspace, normal bound
    for _ in range(2):
        O = Guarded((w.B, w.Hq, w.d), torch.bfloat16)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        abi.sparda_sparse_attn_decode(p, Q, K, V, bg, blk, didx, abi.SPARDA_ADDR_LOGICAL, O.t,
                                      ws.t, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        check_attention(host_bits(O.check("O")).reshape(w.B, 1, w.Hq, w.d), ora,
                        "after timeouts, split=%d" % split)


def test_prefill_waits_run_out_then_the_workspace_serves_the_next_call():
    """The prefill instance of the kernel (K and V tiles refilled
    separately, pairs streamed group by group) under the same one-cycle
    bound."""
    rng = W.rng_for(43)
    B, G, R, d, k, T, nq = 2, 2, 4, 128, 8, 4096 + 29, 96
    Hq = G * R
    Q = W.normal_bf16(rng, (B, nq, Hq, d))
    K = W.normal_bf16(rng, (B, G, T, d))
    V = W.normal_bf16(rng, (B, G, T, d))
    F = W.normal_bf16(rng, (B, nq, G, 1, d))
    _, kcb = oracle.compress_keys(K)
    idx, _, _ = oracle.select(F, kcb, k, 1, 2, T - nq)
    ora = oracle.sparse_attention(Q, K, V, idx, T - nq, T)
    p = abi.make_params(B, Hq, G, T, k)
    p_short = abi.make_params(B, Hq, G, T, k, tune={"attn_wait_cycles": 1})
    ws = Guarded((abi.sparda_workspace_size(abi.SPARDA_OP_ATTN_PREFILL, p, nq),), torch.uint8,
                 fill=0)
    dQ, dK, dV, didx = dev_bf16(Q), dev_bf16(K), dev_bf16(V), torch.from_numpy(idx).cuda()
    timeouts = 0
    for _ in range(3):
        O = torch.empty(B, nq, Hq, d, dtype=torch.bfloat16, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        abi.sparda_sparse_attn_prefill(p_short, dQ, nq, T - nq, dK, dV, T * d, d, didx, O, ws.t, st)
        torch.cuda.synchronize()
        word = int(st.item())
        assert word & ~abi.SPARDA_DEV_TIMEOUT == 0, word
        timeouts += word == abi.SPARDA_DEV_TIMEOUT
    assert timeouts > 0
    ws.check("workspace after timeouts")
    O = Guarded((B, nq, Hq, d), torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.sparda_sparse_attn_prefill(p, dQ, nq, T - nq, dK, dV, T * d, d, didx, O.t, ws.t, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_attention(host_bits(O.check("O")), ora, "prefill after timeouts")
