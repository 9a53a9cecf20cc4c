"""The allocation-free decode attention entry point.

Some callers cannot allocate device memory (for example code running while a
CUDA graph is captured, or a runtime that owns all device memory).  The
library gives them sparda_sparse_attn_decode_noalloc, which keeps its scratch
in a fixed array inside the library.  This file checks, through the C ABI,
that two calls in a row produce what the workspace-taking entry point
produces, and that shapes too large for the fixed scratch are refused.  It is
named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_sparda_b200 import abi, build
from block_sparse_long_sparda_b200 import workloads as W
from tests.parity import check_attention, dev_bf16, host_bits

pytestmark = pytest.mark.gpu


def _case():
    w = W.WORKLOADS["decode_b4_t32k_planted"]
    x = W.decode_inputs(w)
    _, kcb = oracle.compress_keys(x["K"])
    idx, _, _ = oracle.select(x["F"].reshape(w.B, 1, w.G, 1, w.d), kcb, w.k, w.n_init, w.n_local,
                              w.T - 1)
    return w, x, idx[:, 0]


def test_noalloc_decode_matches_workspace_entry_point_twice():
    build.build()
    w, x, idx = _case()
    p = abi.make_params(w.B, w.Hq, w.G, w.T, w.k, w.n_init, w.n_local)
    Q, K, V = dev_bf16(x["Q"]), dev_bf16(x["K"]), dev_bf16(x["V"])
    didx = torch.from_numpy(np.ascontiguousarray(idx)).cuda()
    bg, blk = w.T * w.d, 64 * w.d
    ref = torch.empty(w.B, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
    abi.sparda_sparse_attn_decode(p, Q, K, V, bg, blk, didx, abi.SPARDA_ADDR_LOGICAL, ref,
                                  abi.workspace(abi.SPARDA_OP_ATTN_DECODE, p))
    torch.cuda.synchronize()
    ref_bits = host_bits(ref)
    for _ in range(2):
        out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        abi.sparda_sparse_attn_decode_noalloc(p, Q, K, V, bg, blk, didx, abi.SPARDA_ADDR_LOGICAL,
                                              out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got = host_bits(out)
        check_attention(got, W.bf16_bits_to_f32(ref_bits).astype(np.float64), "noalloc vs workspace")


def test_noalloc_decode_with_lengths_matches_workspace_entry_point():
    """Per-sequence lengths take the same path through both entry points:
    equal outputs, and blocks past a sequence's end flagged by both."""
    build.build()
    w, x, idx = _case()
    sl = torch.tensor([w.T, w.T - 1000 + 7, 500, 0], dtype=torch.int32, device="cuda")
    p = abi.make_params(w.B, w.Hq, w.G, w.T, w.k, w.n_init, w.n_local, seq_len=sl)
    Q, K, V = dev_bf16(x["Q"]), dev_bf16(x["K"]), dev_bf16(x["V"])
    didx = torch.from_numpy(np.ascontiguousarray(idx)).cuda()
    bg, blk = w.T * w.d, 64 * w.d
    ref = torch.empty(w.B, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
    st_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.sparda_sparse_attn_decode(p, Q, K, V, bg, blk, didx, abi.SPARDA_ADDR_LOGICAL, ref,
                                  abi.workspace(abi.SPARDA_OP_ATTN_DECODE, p), st_ref)
    out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.sparda_sparse_attn_decode_noalloc(p, Q, K, V, bg, blk, didx, abi.SPARDA_ADDR_LOGICAL, out,
                                          st)
    torch.cuda.synchronize()
    assert int(st.item()) == int(st_ref.item()) and abi.sparda_status_from_device(int(st.item())) == abi.SPARDA_ERANGE
    check_attention(host_bits(out), W.bf16_bits_to_f32(host_bits(ref)).astype(np.float64),
                    "noalloc vs workspace, lengths")
    assert torch.all(out[3] == 0)


def test_noalloc_decode_refuses_shapes_beyond_its_scratch():
    build.build()
    # enough (query, group) pairs that the partial outputs outgrow the fixed array
    p = abi.make_params(B=4096, Hq=32, G=8, T=131072, k=64)
    assert abi.sparda_workspace_size(abi.SPARDA_OP_ATTN_DECODE, p) > abi.NOALLOC_SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    didx = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(abi.SpardaError) as e:
        abi.sparda_sparse_attn_decode_noalloc(p, dummy, dummy, dummy, 131072 * 128, 64 * 128, didx,
                                              abi.SPARDA_ADDR_LOGICAL, dummy)
    assert e.value.status == abi.SPARDA_EWORKSPACE
