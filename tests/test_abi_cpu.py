"""The C-ABI library: it loads without a GPU, exports every entry point the
header declares, and its host-side validation rejects bad arguments before
anything reaches the device.  No compute calls here."""
import ctypes

import pytest

from block_sparse_long_sparda_b200 import abi, build


@pytest.fixture(scope="module")
def L():
    build.build()
    return abi.lib()


def test_every_declared_entry_point_is_exported(L):
    names = abi.header_functions()
    expected = {"sparda_compress_keys", "sparda_forecast_select", "sparda_prefetch_blocks",
                "sparda_sparse_attn_decode", "sparda_sparse_attn_prefill",
                "sparda_workspace_size", "sparda_status_string", "sparda_status_from_device",
                "sparda_version"}
    assert expected <= set(names)
    for n in names:
        assert hasattr(L, n), n
        assert n in abi._SIGS, "binding lacks " + n


def test_status_strings_and_device_word(L):
    for st in range(0, -7, -1):
        assert abi.sparda_status_string(st).startswith("SPARDA")
    assert abi.sparda_status_from_device(0) == abi.SPARDA_OK
    assert abi.sparda_status_from_device(abi.SPARDA_DEV_RANGE) == abi.SPARDA_ERANGE
    assert abi.sparda_status_from_device(abi.SPARDA_DEV_TIMEOUT | abi.SPARDA_DEV_RANGE) == abi.SPARDA_ETIMEOUT
    assert abi.sparda_status_from_device(abi.SPARDA_DEV_LAYOUT) == abi.SPARDA_ECUDA
    assert abi.sparda_version() >= 100


def _status(fn, *args):
    return getattr(abi.lib(), fn)(*args)


NULL = None


def test_validation_rejects_before_launch(L):
    p = abi.make_params(B=2, Hq=32, G=8, T=4096, k=8)
    byref = ctypes.byref
    fake = ctypes.c_void_p(0x10000)          # aligned, never dereferenced: validation fails first
    odd = ctypes.c_void_p(0x10008)           # 8-byte aligned only
    # unsupported head dim / block size / group ratio
    for bad in (abi.make_params(2, 32, 8, 4096, 8, d=64), abi.make_params(2, 32, 8, 4096, 8, blk=32),
                abi.make_params(2, 24, 8, 4096, 8)):
        st = _status("sparda_compress_keys", byref(bad), fake, 4096 * 128, 128, fake, NULL, NULL)
        assert st in (abi.SPARDA_EUNSUPPORTED,), st
    # Hq not a multiple of G
    st = _status("sparda_compress_keys", byref(abi.make_params(2, 30, 8, 4096, 8)), fake, 1, 128, fake, NULL, NULL)
    assert st == abi.SPARDA_EINVAL
    # null inputs, no outputs, misaligned pointer, bad stride
    assert _status("sparda_compress_keys", byref(p), NULL, 4096 * 128, 128, fake, NULL, NULL) == abi.SPARDA_EINVAL
    assert _status("sparda_compress_keys", byref(p), fake, 4096 * 128, 128, NULL, NULL, NULL) == abi.SPARDA_EINVAL
    assert _status("sparda_compress_keys", byref(p), odd, 4096 * 128, 128, fake, NULL, NULL) == abi.SPARDA_EINVAL
    assert _status("sparda_compress_keys", byref(p), fake, 4096 * 128, 100, fake, NULL, NULL) == abi.SPARDA_EINVAL
    # select: query positions outside the sequence, too many scoring vectors
    assert _status("sparda_forecast_select", byref(p), fake, 1, 1, 4096, fake, fake, NULL, 0, NULL, NULL) == abi.SPARDA_EINVAL
    assert _status("sparda_forecast_select", byref(p), fake, 0, 1, 0, fake, fake, NULL, 0, NULL, NULL) == abi.SPARDA_EINVAL
    assert _status("sparda_forecast_select", byref(p), fake, 1, 17, 4095, fake, fake, NULL, 0, NULL, NULL) == abi.SPARDA_EUNSUPPORTED
    # a multi-chunk select without its workspace
    big = abi.make_params(B=16, Hq=32, G=8, T=131072, k=64)
    assert abi.sparda_workspace_size(abi.SPARDA_OP_SELECT, big, 1, 1) > 0
    assert _status("sparda_forecast_select", byref(big), fake, 1, 1, 131071, fake, fake, NULL, 0, NULL, NULL) == abi.SPARDA_EWORKSPACE
    # decode attention: bad address mode, bad block stride
    assert _status("sparda_sparse_attn_decode", byref(p), fake, fake, fake, 4096 * 128, 64 * 128, fake, 7,
                   fake, NULL, 0, NULL, NULL) == abi.SPARDA_EINVAL
    assert _status("sparda_sparse_attn_decode", byref(p), fake, fake, fake, 4096 * 128, 63 * 128, fake, 0,
                   fake, NULL, 0, NULL, NULL) == abi.SPARDA_EINVAL
    # prefill: rows of a block must be contiguous in this version
    assert _status("sparda_sparse_attn_prefill", byref(p), fake, 16, 4000, fake, fake, 4096 * 256, 256, fake,
                   fake, NULL, 0, NULL, NULL) == abi.SPARDA_EUNSUPPORTED
    # prefetch: negative CTA count
    assert _status("sparda_prefetch_blocks", byref(p), fake, fake, fake, 1, -1, NULL, NULL) == abi.SPARDA_EINVAL
    # empty batch is a valid no-op
    empty = abi.make_params(B=0, Hq=32, G=8, T=4096, k=8)
    assert _status("sparda_compress_keys", byref(empty), NULL, 0, 128, NULL, NULL, NULL) == abi.SPARDA_OK
    # an empty block set is not a valid request
    none = abi.make_params(B=1, Hq=8, G=2, T=4096, k=0, n_init=0, n_local=0)
    assert _status("sparda_compress_keys", byref(none), fake, 4096 * 128, 128, fake, NULL, NULL) == abi.SPARDA_EINVAL


def test_cached_selection_validates_before_touching_the_device(L):
    """sparda_forecast_select_cached rejects bad shapes and arguments on the
    host: a query outside the sequence, too many scoring vectors, fewer slots
    than list entries, missing buffers; an empty batch is a no-op."""
    byref = ctypes.byref
    fake = ctypes.c_void_p(0x10000)
    p = abi.make_params(B=2, Hq=32, G=8, T=4096, k=8)      # S = 11

    def call(prm, nf=1, q_start=4095, C=16, host=fake, idx=fake):
        return _status("sparda_forecast_select_cached", byref(prm), fake, nf, q_start, fake, idx,
                       NULL, 0, C, fake, fake, fake, fake, host, fake, NULL, NULL)
    assert call(p, q_start=4096) == abi.SPARDA_EINVAL
    assert call(p, nf=0) == abi.SPARDA_EINVAL
    assert call(p, nf=17) == abi.SPARDA_EUNSUPPORTED
    assert call(p, C=10) == abi.SPARDA_EINVAL                 # C < S
    assert call(p, C=5000) == abi.SPARDA_EINVAL               # more slots than supported
    assert call(p, idx=NULL) == abi.SPARDA_EINVAL
    assert call(p, host=NULL) == abi.SPARDA_EINVAL
    bad_tune = abi.make_params(B=2, Hq=32, G=8, T=4096, k=8, tune={"attn_stages": 5})
    assert call(bad_tune) == abi.SPARDA_EINVAL
    empty = abi.make_params(B=0, Hq=32, G=8, T=4096, k=8)
    assert call(empty) == abi.SPARDA_OK


def test_workspace_sizes_scale_with_shapes(L):
    small = abi.make_params(B=1, Hq=16, G=2, T=4096, k=4)
    assert abi.sparda_workspace_size(abi.SPARDA_OP_SELECT, small, 1, 1) >= 0
    cfg3 = abi.make_params(B=16, Hq=32, G=8, T=131072, k=64)
    dec = abi.sparda_workspace_size(abi.SPARDA_OP_ATTN_DECODE, cfg3)
    assert dec > 0 and dec < 64 << 20
    # the workspace of an op with no scratch is zero
    assert abi.sparda_workspace_size(abi.SPARDA_OP_COMPRESS, cfg3) == 0
    assert abi.sparda_workspace_size(abi.SPARDA_OP_PREFETCH, cfg3) == 0


def test_head_softmax_validation_and_workspace(L):
    """The per-head softmax selector's entry points refuse bad arguments on the
    host, and its workspace is tickets + failure flags + per-chunk (max, sum)
    pairs + one fp32 score per seen row and head.  Sizes without a GPU use the
    default of 148 SMs, so the chunking is the one-wave rule: B*G = 128
    problems -> 2 chunks of 1024 blocks each."""
    byref = ctypes.byref
    fake = ctypes.c_void_p(0x10000)
    p = abi.make_params(B=16, Hq=32, G=8, T=131072, k=64)
    f = abi.lib().sparda_head_softmax_select
    fw = abi.lib().sparda_head_softmax_select_windows
    assert f(byref(p), fake, 4, 131072, 1.0, fake, fake, NULL, 0, NULL, NULL) == abi.SPARDA_EINVAL   # past the end
    assert f(byref(p), fake, 0, 131071, 1.0, fake, fake, NULL, 0, NULL, NULL) == abi.SPARDA_EINVAL   # no heads
    assert f(byref(p), fake, 17, 131071, 1.0, fake, fake, NULL, 0, NULL, NULL) == abi.SPARDA_EUNSUPPORTED
    assert f(byref(p), fake, 4, 131071, float("nan"), fake, fake, NULL, 0, NULL, NULL) == abi.SPARDA_EINVAL
    assert f(byref(p), fake, 4, 131071, 1.0, fake, fake, NULL, 0, NULL, NULL) == abi.SPARDA_EWORKSPACE
    assert fw(byref(p), fake, 4, 131071, 1.0, fake, 64, 16, fake, NULL, 0, NULL,
              NULL) == abi.SPARDA_EUNSUPPORTED
    assert f(byref(abi.make_params(0, 32, 8, 131072, 64)), NULL, 4, 0, 1.0, NULL, NULL, NULL, 0,
             NULL, NULL) == abi.SPARDA_OK                                                   # empty batch
    words = 2 * 512                        # 128 tickets + 128 flags, each rounded to 256 B
    stats = 128 * 2 * 4 * 8                # (max, sum) per problem, chunk and head
    blocks = abi.sparda_workspace_size(abi.SPARDA_OP_HEAD_SOFTMAX, p, 1, 4)
    windows = abi.sparda_workspace_size(abi.SPARDA_OP_HEAD_SOFTMAX_WINDOWS, p, 1, 4)
    assert blocks == words + stats + 128 * 4 * 2048 * 4
    assert windows == words + stats + 128 * 4 * 8192 * 4
    for op in (abi.SPARDA_OP_HEAD_SOFTMAX, abi.SPARDA_OP_HEAD_SOFTMAX_WINDOWS):
        assert abi.sparda_workspace_size(op, p, 2, 4) == 0                          # decode only
    small = abi.make_params(B=1, Hq=4, G=1, T=64 * 70, k=80)                    # k covers every candidate
    assert abi.sparda_workspace_size(abi.SPARDA_OP_HEAD_SOFTMAX, small, 1, 4) == 0


def test_window_grid_validation(L):
    """The window-grid entry points take only the 32/16 grid, check positions
    and query ranges on the host, and want a workspace at multi-chunk sizes."""
    byref = ctypes.byref
    fake = ctypes.c_void_p(0x10000)
    lib = abi.lib()
    p = abi.make_params(B=2, Hq=32, G=8, T=4096, k=8)
    assert lib.sparda_compress_windows(byref(p), fake, 4096 * 128, 128, 64, 32, NULL, fake,
                                       NULL) == abi.SPARDA_EUNSUPPORTED
    assert lib.sparda_compress_windows(byref(p), fake, 4096 * 128, 128, 32, 16, NULL, NULL,
                                       NULL) == abi.SPARDA_EINVAL            # no output
    assert lib.sparda_append_windows(byref(p), 4096, fake, 4096 * 128, 64 * 128, 32, 16, NULL,
                                     fake, NULL) == abi.SPARDA_EINVAL        # pos past the end
    assert lib.sparda_append_windows(byref(p), 100, fake, 4096 * 128, 64 * 128, 32, 8, NULL,
                                     fake, NULL) == abi.SPARDA_EUNSUPPORTED
    assert lib.sparda_forecast_select_windows(byref(p), fake, 1, 1, 4096, fake, 32, 16, fake,
                                              NULL, 0, NULL, NULL) == abi.SPARDA_EINVAL  # query past T
    assert lib.sparda_forecast_select_windows(byref(p), fake, 1, 1, 4095, fake, 16, 16, fake,
                                              NULL, 0, NULL, NULL) == abi.SPARDA_EUNSUPPORTED
    big = abi.make_params(B=16, Hq=32, G=8, T=131072, k=64)
    assert abi.sparda_workspace_size(abi.SPARDA_OP_SELECT_WINDOWS, big, 1, 1) > 0
    assert lib.sparda_forecast_select_windows(byref(big), fake, 1, 1, 131071, fake, 32, 16, fake,
                                              NULL, 0, NULL, NULL) == abi.SPARDA_EWORKSPACE


def test_tuning_fields_are_validated_and_size_the_workspace(L):
    """Launch choices come only from sparda_params.tune: bad values are
    refused on the host, and the workspace sizes follow the tune pointer the
    calls will use (never the environment)."""
    byref = ctypes.byref
    fake = ctypes.c_void_p(0x10000)
    for bad in ({"attn_stages": 5}, {"attn_stages": 4, "attn_split_kv": 1},
                {"select_chunk": -256}, {"attn_ctas": -1}, {"prefetch_ctas": -2},
                {"attn_wait_cycles": -1}):
        p = abi.make_params(B=2, Hq=32, G=8, T=4096, k=8, tune=bad)
        assert _status("sparda_compress_keys", byref(p), fake, 4096 * 128, 128, fake, NULL,
                       NULL) == abi.SPARDA_EINVAL, bad
    base = abi.make_params(B=16, Hq=32, G=8, T=131072, k=64)
    chunked = abi.make_params(B=16, Hq=32, G=8, T=131072, k=64, tune={"select_chunk": 768})
    assert abi.sparda_workspace_size(abi.SPARDA_OP_SELECT, chunked, 1, 1) != \
        abi.sparda_workspace_size(abi.SPARDA_OP_SELECT, base, 1, 1)
    wide = abi.make_params(B=16, Hq=32, G=8, T=131072, k=64, tune={"attn_ctas": 2000})
    assert abi.sparda_workspace_size(abi.SPARDA_OP_ATTN_DECODE, wide) > \
        abi.sparda_workspace_size(abi.SPARDA_OP_ATTN_DECODE, base)


def test_library_sources_read_no_environment():
    """No kernel choice or workspace size may depend on environment
    variables: the library's sources never call getenv."""
    import glob
    import os
    csrc = os.path.join(os.path.dirname(abi.PKG), "block_sparse_long_sparda_b200", "csrc")
    for f in glob.glob(os.path.join(csrc, "*")):
        with open(f) as fh:
            assert "getenv" not in fh.read(), f
