"""The C ABI without a GPU: the library loads, exports every declared entry
point, and rejects bad arguments before touching the device."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def moe():
    import __graft_entry__

    __graft_entry__.build()
    import sparse_moe_layer_07_b200 as m

    return m


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_five_calls():
    names = declared_symbols()
    for n in ("moe_router_topk", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_layer_forward"):
        assert n in names


def test_every_declared_symbol_is_exported(moe):
    lib = ctypes.CDLL(moe.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def _cfg(moe, **kw):
    base = dict(T=64, d=256, f=1024, capacity_factor=1.25, dtype="f32")
    base.update(kw)
    return moe.Config(**base)


def test_status_strings(moe):
    for code, name in moe.STATUS.items():
        assert moe.lib.moe_status_string(code).decode() == name


def test_capacity_matches_oracle(moe):
    import oracle

    for T, cf in [(64, 1.25), (2048, 1.25), (8192, 4.0), (16384, 1.25), (10, 1.0), (7, 0.3), (32, math.inf),
                  (100, 1.1), (1000, 0.01), (5, 100.0)]:
        c = _cfg(moe, T=T, capacity_factor=cf)
        assert moe.capacity(c) == min(oracle.capacity(T, 2, 8, cf), T), (T, cf)


@pytest.mark.parametrize("kw,status", [
    (dict(E=4), "MOE_ERR_UNSUPPORTED"),
    (dict(top_k=1), "MOE_ERR_UNSUPPORTED"),
    (dict(d=100), "MOE_ERR_UNSUPPORTED"),
    (dict(dtype="bf16", f=192), "MOE_ERR_UNSUPPORTED"),
    (dict(capacity_factor=0.0), "MOE_ERR_INVALID_ARG"),
    (dict(capacity_factor=float("nan")), "MOE_ERR_INVALID_ARG"),
    (dict(capacity_factor=-1.0), "MOE_ERR_INVALID_ARG"),
    (dict(T=-1), "MOE_ERR_INVALID_ARG"),
])
def test_bad_config_rejected_before_launch(moe, kw, status):
    c = _cfg(moe, **kw)
    P = ctypes.c_void_p
    fake = P(16)  # never dereferenced: validation fails first
    st = moe.lib.moe_router_topk(c.ref, fake, fake, None, None, fake, fake, None)
    assert moe.STATUS[st] == status
    assert moe.capacity(c) == -1
    assert moe.workspace_size(c) == 0


def test_null_and_misaligned_pointers_rejected(moe):
    c = _cfg(moe)
    P = ctypes.c_void_p
    ok = P(256)
    assert moe.STATUS[moe.lib.moe_router_topk(c.ref, None, ok, None, None, ok, ok, None)] == "MOE_ERR_INVALID_ARG"
    assert moe.STATUS[moe.lib.moe_router_topk(c.ref, P(258), ok, None, None, ok, ok, None)] == "MOE_ERR_INVALID_ARG"
    assert moe.STATUS[moe.lib.moe_combine(c.ref, ok, ok, None, 0, ok, None)] == "MOE_ERR_INVALID_ARG"
    st = moe.lib.moe_layer_forward(c.ref, ok, None, None, ok, ok, ok, ok, None, ok, 1 << 30, None)
    assert moe.STATUS[st] == "MOE_ERR_INVALID_ARG"


def test_small_workspace_rejected(moe):
    c = _cfg(moe, T=4096)
    P = ctypes.c_void_p
    ok = P(256)
    need = moe.dispatch_workspace_size(c)
    assert need >= 16 * 8 * 4
    st = moe.lib.moe_dispatch(c.ref, ok, ok, ok, ok, ok, ok, ok, ok, ok, ok, ok, need - 1, None)
    assert moe.STATUS[st] == "MOE_ERR_WORKSPACE"
    st = moe.lib.moe_layer_forward(c.ref, ok, ok, None, ok, ok, ok, ok, None, ok, moe.workspace_size(c) - 1, None)
    assert moe.STATUS[st] == "MOE_ERR_WORKSPACE"


def test_empty_batch_is_a_no_op(moe):
    c = _cfg(moe, T=0)
    P = ctypes.c_void_p
    ok = P(256)
    assert moe.lib.moe_router_topk(c.ref, None, None, None, None, None, None, None) == 0
    assert moe.lib.moe_layer_forward(c.ref, None, ok, None, ok, ok, ok, None, None, None, 0, None) == 0


def test_workspace_grows_with_tokens(moe):
    a = moe.workspace_size(_cfg(moe, T=64, dtype="bf16"))
    b = moe.workspace_size(_cfg(moe, T=128, dtype="bf16"))
    assert 0 < a < b


def test_noalloc_dispatch_rejects_oversize_before_launch(moe):
    P = ctypes.c_void_p
    ok = P(256)
    big = _cfg(moe, T=moe.NOALLOC_MAX_TOKENS + 1, dtype="bf16", d=256, f=384)
    st = moe.lib.moe_dispatch_noalloc(big.ref, None, ok, ok, ok, ok, ok, ok, ok, ok, None, None)
    assert moe.STATUS[st] == "MOE_ERR_UNSUPPORTED"
    bad = _cfg(moe, E=4)
    assert moe.STATUS[moe.lib.moe_dispatch_noalloc(bad.ref, None, ok, ok, ok, ok, ok, ok, ok, ok, None,
                                                   None)] == "MOE_ERR_UNSUPPORTED"
    small = _cfg(moe, T=64)
    assert moe.STATUS[moe.lib.moe_dispatch_noalloc(small.ref, None, None, ok, ok, ok, ok, ok, ok, ok, None,
                                                   None)] == "MOE_ERR_INVALID_ARG"


def test_host_batches_argument_errors_before_launch(moe):
    c = _cfg(moe, T=64, dtype="bf16")
    P = ctypes.c_void_p
    ok = P(256)
    need = moe.workspace_size_host_batches(c)
    base = moe.workspace_size(c)
    assert need >= base + 2 * 64 * c.d * 2
    arr = (P * 2)(ok, ok)
    holes = (P * 2)(ok, None)
    f = moe.lib.moe_layer_forward_host_batches
    assert moe.STATUS[f(c.ref, -1, arr, ok, None, ok, ok, ok, arr, ok, need, None)] == "MOE_ERR_INVALID_ARG"
    assert moe.STATUS[f(c.ref, 2, None, ok, None, ok, ok, ok, arr, ok, need, None)] == "MOE_ERR_INVALID_ARG"
    assert moe.STATUS[f(c.ref, 2, arr, ok, None, ok, ok, ok, holes, ok, need, None)] == "MOE_ERR_INVALID_ARG"
    # the layer workspace alone is not enough: the second staging slot is missing
    assert moe.STATUS[f(c.ref, 2, arr, ok, None, ok, ok, ok, arr, ok, base, None)] == "MOE_ERR_WORKSPACE"
    assert f(c.ref, 0, None, ok, None, ok, ok, ok, None, ok, need, None) == 0
    assert moe.workspace_size_host_batches(_cfg(moe, E=4)) == 0


def test_down_combine_scope_checked_before_launch(moe):
    P = ctypes.c_void_p
    ok = P(256)
    f32 = _cfg(moe, T=1024, dtype="f32")
    odd = _cfg(moe, T=1024, dtype="bf16", d=384)
    small = _cfg(moe, T=64, dtype="bf16")  # weight-streaming size
    for c in (f32, odd, small):
        assert moe.STATUS[moe.lib.moe_expert_down_combine(c.ref, ok, ok, ok, ok, ok, ok, ok, 1 << 30, None)] == \
            "MOE_ERR_UNSUPPORTED"
    big = _cfg(moe, T=1024, dtype="bf16", d=512)
    need = moe.lib.moe_expert_down_combine_workspace_size(big.ref)
    assert need >= 1024 * 512 * 4
    st = moe.lib.moe_expert_down_combine(big.ref, ok, ok, ok, ok, ok, ok, ok, need - 1, None)
    assert moe.STATUS[st] == "MOE_ERR_WORKSPACE"
    st = moe.lib.moe_expert_down_combine(big.ref, ok, ok, ok, ok, None, ok, ok, need, None)
    assert moe.STATUS[st] == "MOE_ERR_INVALID_ARG"


def test_training_entry_points_checked_before_launch(moe):
    P = ctypes.c_void_p
    ok = P(256)
    f32 = _cfg(moe, T=64, dtype="f32")
    odd = _cfg(moe, T=64, dtype="bf16", d=384, f=512)
    assert moe.workspace_size_train(f32) == 0 and moe.workspace_size_train(odd) == 0
    for c in (f32, odd):
        assert moe.STATUS[moe.lib.moe_layer_forward_train(c.ref, ok, ok, None, ok, ok, ok, ok, ok, 1 << 40,
                                                          None)] == "MOE_ERR_UNSUPPORTED"
        assert moe.STATUS[moe.lib.moe_layer_backward(c.ref, ok, ok, ok, ok, ok, ok, ok, ok, None, ok, ok, ok, ok,
                                                     1 << 40, None)] == "MOE_ERR_UNSUPPORTED"
    c = _cfg(moe, T=64, dtype="bf16", d=256, f=512)
    need = moe.workspace_size_train(c)
    assert need > moe.workspace_size(c)
    st = moe.lib.moe_layer_forward_train(c.ref, ok, ok, None, ok, ok, ok, ok, ok, need - 1, None)
    assert moe.STATUS[st] == "MOE_ERR_WORKSPACE"
    st = moe.lib.moe_layer_backward(c.ref, ok, ok, ok, ok, ok, ok, ok, ok, None, ok, ok, ok, ok, need - 1, None)
    assert moe.STATUS[st] == "MOE_ERR_WORKSPACE"
    st = moe.lib.moe_layer_backward(c.ref, ok, ok, ok, ok, ok, ok, ok, None, None, ok, ok, ok, ok, need, None)
    assert moe.STATUS[st] == "MOE_ERR_INVALID_ARG"


def test_shard_dispatch_arguments_checked_before_launch(moe):
    P = ctypes.c_void_p
    ok = P(256)
    c = _cfg(moe, T=64)
    ws = moe.dispatch_workspace_size(c)
    f = moe.lib.moe_dispatch_shard
    assert moe.STATUS[f(c.ref, 10, ok, 2, 2, None, ok, ok, ok, ok, ok, ok, ok, ok, None, ok, ws, None)] == \
        "MOE_ERR_INVALID_ARG"  # shard index out of range
    assert moe.STATUS[f(c.ref, -1, ok, 2, 0, None, ok, ok, ok, ok, ok, ok, ok, ok, None, ok, ws, None)] == \
        "MOE_ERR_INVALID_ARG"  # negative capacity
    assert moe.STATUS[f(c.ref, 10, None, 2, 0, None, ok, ok, ok, ok, ok, ok, ok, ok, None, ok, ws, None)] == \
        "MOE_ERR_INVALID_ARG"  # no count table
    assert moe.STATUS[f(c.ref, 10, ok, 2, 0, None, ok, ok, ok, ok, ok, ok, ok, ok, None, ok, ws - 1, None)] == \
        "MOE_ERR_WORKSPACE"
    assert moe.STATUS[moe.lib.moe_route_counts(c.ref, ok, None, None)] == "MOE_ERR_INVALID_ARG"


def test_gather_rows_arguments_checked_before_launch(moe):
    P = ctypes.c_void_p
    ok = P(256)
    f = moe.lib.moe_gather_rows
    assert f(ok, 10, ok, 0, 16, ok, None) == 0  # nothing to copy
    assert moe.STATUS[f(ok, 10, ok, 4, 24, ok, None)] == "MOE_ERR_INVALID_ARG"  # row not a multiple of 16 bytes
    assert moe.STATUS[f(ok, 10, ok, -1, 16, ok, None)] == "MOE_ERR_INVALID_ARG"
    assert moe.STATUS[f(None, 10, ok, 4, 16, ok, None)] == "MOE_ERR_INVALID_ARG"
    assert moe.STATUS[f(P(258), 10, ok, 4, 16, ok, None)] == "MOE_ERR_INVALID_ARG"  # misaligned source


def test_bounded_wait_check_limits(moe):
    assert moe.STATUS[moe.lib.moe_check_bounded_wait(10, None)] == "MOE_ERR_INVALID_ARG"
    assert moe.STATUS[moe.lib.moe_check_bounded_wait(2_000_000_000, None)] == "MOE_ERR_INVALID_ARG"


def test_gemm_tile_mode_setting(moe):
    import ctypes

    prev = ctypes.c_int32(-1)
    assert moe.STATUS[moe.lib.moe_set_gemm_tiles(7, ctypes.byref(prev))] == "MOE_ERR_INVALID_ARG"
    assert prev.value == -1  # untouched on error
    assert moe.set_gemm_tiles("pair") == "auto"
    with moe.gemm_tiles("single"):
        assert moe.set_gemm_tiles("single") == "single"
    assert moe.set_gemm_tiles("auto") == "pair"  # the context manager restored "pair"
    assert moe.STATUS[moe.lib.moe_set_gemm_tiles(0, None)] == "MOE_OK"
    with pytest.raises(ValueError):
        moe.set_gemm_tiles("quad")


def test_binding_checks_element_counts_and_types(moe):
    import torch

    c = _cfg(moe, T=4, d=128, f=128, dtype="bf16")
    x = torch.zeros((4, 128), dtype=torch.float32)  # wrong type for a bf16 layer
    wr = torch.zeros((8, 128), dtype=torch.bfloat16)
    w = torch.zeros((8, 128, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="x must be"):
        moe.layer_forward(c, x, wr, w, w, w)
    with pytest.raises(ValueError, match="w_gate must hold"):
        moe.layer_forward(c, x.to(torch.bfloat16), wr, w[:4], w, w)
    with pytest.raises(ValueError, match="logit_bias must be"):
        moe.router_topk(c, x.to(torch.bfloat16), wr, logit_bias=torch.zeros(8, dtype=torch.float64))


def test_utilization_arguments_checked_before_launch(moe):
    p = ctypes.c_void_p(16)  # never dereferenced: the call must fail on E first
    for E in (0, -1, 65):
        assert moe.lib.moe_expert_utilization(p, E, p, p, None) == 1  # MOE_ERR_INVALID_ARG
    assert moe.lib.moe_expert_utilization(None, 8, p, p, None) == 1
    assert moe.lib.moe_expert_utilization(p, 8, None, p, None) == 1
    assert moe.lib.moe_expert_utilization(p, 8, p, None, None) == 1


def test_phase_profile_read_without_events(moe):
    """With nothing recorded, a read fills zeros for the phases asked for, takes
    NULL arrays and shorter arrays, and rejects a negative count."""
    assert moe.PHASES[7] == "bwd_dh" and len(moe.PHASES) == 14
    moe.profile_phases(True)
    try:
        got = moe.profile_read()
        assert set(got) == set(moe.PHASES) and all(v == (0.0, 0) for v in got.values())
        ms = (ctypes.c_float * 3)(9.0, 9.0, 9.0)
        calls = (ctypes.c_int32 * 3)(7, 7, 7)
        assert moe.lib.moe_profile_read(ms, calls, 3) == 0
        assert list(ms) == [0.0, 0.0, 0.0] and list(calls) == [0, 0, 0]
        assert moe.lib.moe_profile_read(None, None, 14) == 0
        assert moe.lib.moe_profile_read(ms, calls, -1) == 1
    finally:
        moe.profile_phases(False)


def test_peer_entry_points_check_arguments_before_any_cuda_call():
    # every case below is rejected on the host before the library touches CUDA,
    # so fake device addresses are never dereferenced
    import ctypes

    from sparse_moe_layer_07_b200 import Config, EpPeers, lib

    cfg = Config(512, 256, 384)
    good = [(0x10000 * (q + 1), 0x100000 + 0x1000 * q, 0x200000 + 0x1000 * q, 0x300000 + 0x1000 * q)
            for q in range(2)]
    fake = ctypes.c_void_p(0x400000)

    def dispatch(peers, c=cfg):
        return lib.moe_ep_dispatch_peers(c.ref, peers.ref, fake, fake, fake, fake, fake, fake, None)

    def ffn(peers, c=cfg):
        return lib.moe_ep_expert_ffn_peers(c.ref, peers.ref, fake, fake, fake, fake, fake, None)

    def combine(peers, c=cfg):
        return lib.moe_ep_combine_peers(c.ref, peers.ref, fake, None)

    def with_part(q, k, delta):
        rows = [list(r) for r in good]
        rows[q][k] += delta
        return EpPeers(2, 0, [tuple(r) for r in rows])

    for call in (dispatch, ffn, combine):
        assert call(with_part(1, 1, 2)) == 1      # src not 4-byte aligned
        assert call(with_part(0, 2, 1)) == 1      # scale not 4-byte aligned
        assert call(with_part(1, 0, 8)) == 1      # x_grp not 16-byte aligned
        assert call(with_part(0, 3, 4)) == 1      # sums not 16-byte aligned
        assert call(with_part(1, 3, -good[1][3])) == 1  # a NULL buffer
        assert call(EpPeers(3, 0, good + [good[0]])) == 2  # 3 ranks do not divide E = 8
        assert call(EpPeers(2, 0, good), Config(512, 256, 384, dtype="f32")) == 2
        assert call(EpPeers(2, 0, good), Config(512, 128, 384)) == 2  # d not a multiple of 256
