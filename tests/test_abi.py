"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before launching anything.
No GPU is needed (no call here reaches a CUDA launch)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def B():
    from sigmoid_top_routing_warp_b200 import build
    build.build()
    from sigmoid_top_routing_warp_b200 import binding
    return binding


def header_functions():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b((?:moe|dsa)_[a-z_]+)\s*\(", src))
    return sorted(names)


def test_every_declared_symbol_is_exported(B):
    names = header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(B.lib(), n), n
    assert sorted(B.EXPORTED) == names


def cfg(B, **kw):
    base = dict(T=64, H=5120, E=256, k=8, I=1536, n_shared=1)
    base.update(kw)
    return B.MoeConfig(**base)


def test_workspace_size_and_offsets(B):
    c = cfg(B)
    n = B.workspace_size(c)
    T, E, k, H, I = 64, 256, 8, 5120, 1536
    # at least the gathered activations, intermediates and outputs
    assert n >= T * k * H * 2 * 2 + T * k * I * 2 + T * H * 2
    offs = [B.workspace_offset(c, it) for it in B.WS_ITEMS]
    assert all(o % 256 == 0 and o < n for o in offs)
    assert len(set(offs)) == len(offs)
    big = cfg(B, T=8192)
    assert B.workspace_size(big) > n
    # the routed outputs y hold fp32 rows when k = 1, bf16 otherwise: the next
    # region starts at least T*k*H*4 (resp. *2) bytes after y
    for kk, el in ((1, 4), (2, 2)):
        c1 = cfg(B, k=kk)
        y0, ysh0 = B.workspace_offset(c1, "y"), B.workspace_offset(c1, "y_shared")
        assert ysh0 - y0 >= T * kk * H * el


@pytest.mark.parametrize("kw", [dict(H=100), dict(E=33), dict(E=0), dict(k=0), dict(k=300),
                                dict(I=100), dict(n_group=3), dict(n_group=8, topk_group=9),
                                dict(n_group=8, topk_group=1, k=33), dict(T=-1), dict(dtype=7),
                                dict(n_shared=-1), dict(flags=0x80)])
def test_invalid_configs_rejected(B, kw):
    with pytest.raises(B.MoeError):
        B.workspace_size(cfg(B, **kw))
    assert B.get_last_error() != ""


def test_calls_reject_bad_arguments_before_launch(B):
    c = cfg(B)
    cc = c.c()
    ws_bytes = B.workspace_size(c)
    fake_ws = 1 << 20  # aligned, never dereferenced: validation fails first
    L = B.lib()
    st = L.moe_route(ctypes.byref(cc), None, None, None, None, None, None, fake_ws, ws_bytes,
                     None)
    assert st == B.MOE_ERR_INVALID_ARG and "x" in B.get_last_error()
    st = L.moe_route(ctypes.byref(cc), 16, 16, 16, 16, 16, 16, fake_ws, ws_bytes - 1, None)
    assert st == B.MOE_ERR_WORKSPACE
    st = L.moe_route(ctypes.byref(cc), 16, 16, 16, 16, 16, 16, fake_ws + 8, ws_bytes, None)
    assert st == B.MOE_ERR_INVALID_ARG and "aligned" in B.get_last_error()
    st = L.moe_permute(ctypes.byref(cc), None, 16, 16, 16, fake_ws, ws_bytes, None)
    assert st == B.MOE_ERR_INVALID_ARG
    st = L.moe_combine(ctypes.byref(cc), 24, 16, None, 32, None)   # y misaligned
    assert st == B.MOE_ERR_INVALID_ARG and "aligned" in B.get_last_error()
    st = L.moe_forward(ctypes.byref(cc), *([16] * 4), 16, *([16] * 7), fake_ws, ws_bytes, None,
                       None)  # a weight scale given for bf16 weights
    assert st == B.MOE_ERR_INVALID_ARG and "scale" in B.get_last_error()
    st = L.moe_forward(None, *([16] * 12), fake_ws, ws_bytes, None, None)
    assert st == B.MOE_ERR_INVALID_ARG
    st = L.moe_check_device_status(None, None)
    assert st == B.MOE_ERR_INVALID_ARG


def test_bias_update_rejects_bad_arguments_before_launch(B):
    L = B.lib()
    cc = cfg(B).c()
    for g in (float("nan"), -1.0, float("inf")):
        st = L.moe_bias_update(ctypes.byref(cc), None, None, g, None)
        assert st == B.MOE_ERR_INVALID_ARG and "gamma" in B.get_last_error()
    st = L.moe_bias_update(ctypes.byref(cc), None, 16, 1e-3, None)
    assert st == B.MOE_ERR_INVALID_ARG and "topk_idx" in B.get_last_error()
    st = L.moe_bias_update(ctypes.byref(cc), 16, None, 1e-3, None)
    assert st == B.MOE_ERR_INVALID_ARG and "bias" in B.get_last_error()
    bad = cfg(B, E=33).c()
    assert L.moe_bias_update(ctypes.byref(bad), 16, 16, 1e-3, None) != B.MOE_OK
    # T = 0: nothing to count, nothing launched
    empty = cfg(B, T=0).c()
    assert L.moe_bias_update(ctypes.byref(empty), 16, 16, 1e-3, None) == B.MOE_OK


def test_empty_batch_is_a_no_op(B):
    c = cfg(B, T=0)
    cc = c.c()
    ws_bytes = B.workspace_size(c)
    st = B.lib().moe_forward(ctypes.byref(cc), 16, 16, 16, 16, None, 16, None, 16, None, 16,
                             None, 16, 1 << 20, ws_bytes, None, None)
    assert st == B.MOE_OK


def test_block_and_norm_reject_bad_arguments_before_launch(B):
    c = cfg(B)
    cc = c.c()
    ws_bytes = B.workspace_size(c)
    fake_ws = 1 << 20
    L = B.lib()
    st = L.moe_rmsnorm(ctypes.byref(cc), 16, None, ctypes.c_float(1e-6), 1 << 30, None)
    assert st == B.MOE_ERR_INVALID_ARG and "gamma" in B.get_last_error()
    st = L.moe_rmsnorm(ctypes.byref(cc), 16, 16, ctypes.c_float(-1.0), 1 << 30, None)
    assert st == B.MOE_ERR_INVALID_ARG and "eps" in B.get_last_error()
    st = L.moe_rmsnorm(ctypes.byref(cc), 16, 16, ctypes.c_float(float("nan")), 1 << 30, None)
    assert st == B.MOE_ERR_INVALID_ARG and "eps" in B.get_last_error()
    st = L.moe_rmsnorm(ctypes.byref(cc), 1 << 20, 16, ctypes.c_float(1e-6), (1 << 20) + 4096,
                       None)  # u overlaps h
    assert st == B.MOE_ERR_INVALID_ARG and "overlap" in B.get_last_error()
    bad = cfg(B, H=100).c()
    st = L.moe_rmsnorm(ctypes.byref(bad), 16, 16, ctypes.c_float(1e-6), 1 << 30, None)
    assert st == B.MOE_ERR_INVALID_ARG
    args = [16] * 12
    st = L.moe_forward_block(ctypes.byref(cc), 16, None, ctypes.c_float(1e-6), *args, fake_ws,
                             ws_bytes, None, None)
    assert st == B.MOE_ERR_INVALID_ARG and "gamma" in B.get_last_error()
    st = L.moe_forward_block(ctypes.byref(cc), 1 << 24, 16, ctypes.c_float(1e-6),
                             16, 16, 16, None, 16, None, 16, None, 16, None, (1 << 24) + 64,
                             fake_ws, ws_bytes, None, None)  # out partly overlaps h
    assert st == B.MOE_ERR_INVALID_ARG and "overlap" in B.get_last_error()
    st = L.moe_forward_block(ctypes.byref(cc), 16, 16, ctypes.c_float(1e-6),
                             16, 16, 16, None, 16, None, 16, None, 16, None, 16,
                             fake_ws, ws_bytes - 1, None, None)
    assert st == B.MOE_ERR_WORKSPACE
    # empty batch: validated, nothing launched
    c0 = cfg(B, T=0).c()
    st = L.moe_forward_block(ctypes.byref(c0), 16, 16, ctypes.c_float(1e-6),
                             16, 16, 16, None, 16, None, 16, None, 16, None, 16,
                             fake_ws, B.workspace_size(cfg(B, T=0)), None, None)
    assert st == B.MOE_OK


def test_dsa_calls_reject_bad_arguments_before_launch(B):
    c = B.DsaConfig(Sq=64, Sk=1024)
    cc = c.c()
    L = B.lib()
    n = B.dsa_workspace_size(c)
    assert n >= 64 * 1024 * 4 and L.dsa_workspace_scores_offset() % 256 == 0
    for bad in (dict(head_dim=64), dict(topk=0), dict(topk=4096), dict(n_heads=0),
                dict(Sq=-1), dict(q_offset=-3)):
        kw = dict(Sq=64, Sk=1024)
        kw.update(bad)
        with pytest.raises(B.MoeError):
            B.dsa_workspace_size(B.DsaConfig(**kw))
    raw = B.DsaConfigC(64, 1024, 64, 128, 2048, 2, 0, 1)  # causal must be 0 or 1
    assert L.dsa_workspace_size(ctypes.byref(raw)) == 0 and "causal" in B.get_last_error()
    st = L.dsa_index_scores(ctypes.byref(cc), None, 16, 16, 16, 1 << 20, 256, None)
    assert st == B.MOE_ERR_INVALID_ARG and "q" in B.get_last_error()
    st = L.dsa_index_scores(ctypes.byref(cc), 24, 16, 16, 16, 1 << 20, 256, None)
    assert st == B.MOE_ERR_INVALID_ARG and "aligned" in B.get_last_error()
    st = L.dsa_indexer(ctypes.byref(cc), 16, 16, 16, 16, 1 << 20, n - 1, None)
    assert st == B.MOE_ERR_WORKSPACE
    st = L.dsa_index_topk(ctypes.byref(cc), None, 16, None)
    assert st == B.MOE_ERR_INVALID_ARG
    hd = B.DsaConfig(Sq=4, Sk=4, head_dim=64).c()
    st = L.dsa_index_topk(ctypes.byref(hd), 16, 16, None)
    assert st == B.MOE_ERR_UNSUPPORTED


def test_backward_rejects_bad_arguments_before_launch(B):
    """moe_backward validates on the host: fp8 layers, NULL or misaligned
    buffers and a short workspace are refused before anything is launched."""
    c = cfg(B)
    cc = c.c()
    n = B.backward_workspace_size(c)
    # the padded row buffers: at least the gathered rows of x and dout, the
    # gate/up pre-activations and their gradients
    assert n >= 2 * 64 * 8 * 5120 * 2 + 2 * 64 * 8 * 3072 * 2
    assert B.backward_workspace_size(cfg(B, T=8192)) > n
    L = B.lib()
    p = 1 << 20  # aligned, never dereferenced
    args = [p] * 17  # x .. dlogits; every call below fails validation, none launches
    fp8 = cfg(B, dtype=B.MOE_DTYPE_FP8_E4M3_BLOCK128).c()
    assert L.moe_backward(ctypes.byref(fp8), *args, p, n, None, None) == B.MOE_ERR_UNSUPPORTED
    bad = list(args)
    bad[9] = None  # dout
    assert L.moe_backward(ctypes.byref(cc), *bad, p, n, None, None) == B.MOE_ERR_INVALID_ARG
    assert "dout" in B.get_last_error()
    bad = list(args)
    bad[10] = p + 2  # dx misaligned
    assert L.moe_backward(ctypes.byref(cc), *bad, p, n, None, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_backward(ctypes.byref(cc), *args, p, n - 256, None, None) == B.MOE_ERR_WORKSPACE
    assert L.moe_backward(ctypes.byref(cc), *args, p + 128, n, None, None) == B.MOE_ERR_INVALID_ARG
