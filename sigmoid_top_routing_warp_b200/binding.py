"""ctypes binding of libmoe_b200.so (the C ABI in include/moe.h).

Argument marshalling only: torch tensors are passed as raw device pointers
together with the current CUDA stream; every step of the layer runs in the
library's kernels.  There is no fallback: if the shared library is missing,
importing this module raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError("libmoe_b200.so is not built (%s); build it with "
                      "`python -m sigmoid_top_routing_warp_b200.build`" % _LIB_PATH)
_lib = ctypes.CDLL(_LIB_PATH)

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, \
    MOE_ERR_TIMEOUT = range(6)
MOE_DTYPE_BF16 = 0
MOE_DTYPE_FP8_E4M3_BLOCK128 = 1
MOE_NUM_STAGES = 6
MOE_NUM_BWD_STAGES = 7
BWD_STAGE_NAMES = ("dispatch", "gate_up_recompute", "down_backward", "router", "input_grads",
                   "weight_grads", "combine")
MOE_FLAG_TEST_STALL = 0x1
STAGE_NAMES = ("router_gemm", "router_select", "dispatch", "gate_up_swiglu", "down_weighted",
               "combine")
WS_ITEMS = {"logits": 0, "topk_idx": 1, "topk_w": 2, "offsets": 3, "rows": 4, "pos": 5,
            "y": 6, "y_shared": 7, "u": 8}

# Every symbol include/moe.h declares.
EXPORTED = ("moe_get_last_error", "moe_workspace_size", "moe_workspace_offset", "moe_route",
            "moe_route_from_logits", "moe_bias_update", "moe_permute", "moe_expert_ffn",
            "moe_combine", "moe_forward", "moe_check_device_status", "moe_permute_noalloc",
            "moe_quantize_act", "moe_rmsnorm", "moe_forward_block",
            "moe_backward_workspace_size", "moe_backward", "moe_ep_pack",
            "moe_shared_expert", "moe_ep_expert_counts", "moe_ep_plan", "moe_ep_dispatch_peer",
            "moe_ep_combine_peer",
            "dsa_workspace_size", "dsa_workspace_scores_offset", "dsa_index_scores",
            "dsa_index_topk", "dsa_indexer")


class MoeConfigC(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("I", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
                ("group_topn", ctypes.c_int32), ("norm_topk_prob", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


@dataclass
class MoeConfig:
    """moe_config_t (field names follow the Dots1 / DeepSeek-V3 config)."""
    T: int
    H: int
    E: int
    k: int
    I: int
    n_shared: int = 1
    n_group: int = 1
    topk_group: int = 1
    group_topn: int = 2
    norm_topk_prob: bool = True
    routed_scaling_factor: float = 1.0
    dtype: int = MOE_DTYPE_BF16
    flags: int = 0

    def c(self) -> MoeConfigC:
        return MoeConfigC(self.T, self.H, self.E, self.k, self.I, self.n_shared, self.n_group,
                          self.topk_group, self.group_topn, int(bool(self.norm_topk_prob)),
                          float(self.routed_scaling_factor), self.dtype, self.flags)

    @property
    def Is(self) -> int:
        return self.n_shared * self.I


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed (status %d): %s" % (where, status, get_last_error()))


_P = ctypes.c_void_p
_CFG = ctypes.POINTER(MoeConfigC)
_lib.moe_get_last_error.restype = ctypes.c_char_p
_lib.moe_get_last_error.argtypes = []
_lib.moe_workspace_size.restype = ctypes.c_size_t
_lib.moe_workspace_size.argtypes = [_CFG]
_lib.moe_workspace_offset.restype = ctypes.c_size_t
_lib.moe_workspace_offset.argtypes = [_CFG, ctypes.c_int32]
_lib.moe_route.restype = ctypes.c_int
_lib.moe_route.argtypes = [_CFG, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_route_from_logits.restype = ctypes.c_int
_lib.moe_route_from_logits.argtypes = [_CFG, _P, _P, _P, _P, _P]
_lib.moe_bias_update.restype = ctypes.c_int
_lib.moe_bias_update.argtypes = [_CFG, _P, _P, ctypes.c_float, _P]
_lib.moe_permute.restype = ctypes.c_int
_lib.moe_permute.argtypes = [_CFG, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_expert_ffn.restype = ctypes.c_int
_lib.moe_expert_ffn.argtypes = [_CFG] + [_P] * 16 + [ctypes.c_size_t, _P]
_lib.moe_combine.restype = ctypes.c_int
_lib.moe_combine.argtypes = [_CFG, _P, _P, _P, _P, _P]
_lib.moe_forward.restype = ctypes.c_int
_lib.moe_forward.argtypes = [_CFG] + [_P] * 13 + [ctypes.c_size_t, _P, _P]


class DsaConfigC(ctypes.Structure):
    _fields_ = [("Sq", ctypes.c_int32), ("Sk", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("topk", ctypes.c_int32), ("causal", ctypes.c_int32),
                ("q_offset", ctypes.c_int32), ("sorted", ctypes.c_int32)]


_DCFG = ctypes.POINTER(DsaConfigC)
_lib.dsa_workspace_size.restype = ctypes.c_size_t
_lib.dsa_workspace_size.argtypes = [_DCFG]
_lib.dsa_workspace_scores_offset.restype = ctypes.c_size_t
_lib.dsa_workspace_scores_offset.argtypes = []
_lib.dsa_index_scores.restype = ctypes.c_int
_lib.dsa_index_scores.argtypes = [_DCFG, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.dsa_index_topk.restype = ctypes.c_int
_lib.dsa_index_topk.argtypes = [_DCFG, _P, _P, _P]
_lib.dsa_indexer.restype = ctypes.c_int
_lib.dsa_indexer.argtypes = [_DCFG, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_rmsnorm.restype = ctypes.c_int
_lib.moe_rmsnorm.argtypes = [_CFG, _P, _P, ctypes.c_float, _P, _P]
_lib.moe_forward_block.restype = ctypes.c_int
_lib.moe_forward_block.argtypes = ([_CFG, _P, _P, ctypes.c_float] + [_P] * 12 +
                                   [ctypes.c_size_t, _P, _P])
_lib.moe_permute_noalloc.restype = ctypes.c_int
_lib.moe_permute_noalloc.argtypes = [_CFG, _P, _P, _P, _P, _P]
_lib.moe_quantize_act.restype = ctypes.c_int
_lib.moe_quantize_act.argtypes = [_P, ctypes.c_int32, ctypes.c_int32, _P, _P, _P]
_lib.moe_backward_workspace_size.restype = ctypes.c_size_t
_lib.moe_backward_workspace_size.argtypes = [_CFG]
_lib.moe_backward.restype = ctypes.c_int
_lib.moe_backward.argtypes = [_CFG] + [_P] * 18 + [ctypes.c_size_t, _P, _P]
_lib.moe_ep_pack.restype = ctypes.c_int
_lib.moe_ep_pack.argtypes = [_CFG, ctypes.c_int32] + [_P] * 10
_lib.moe_shared_expert.restype = ctypes.c_int
_lib.moe_shared_expert.argtypes = [_CFG] + [_P] * 5 + [ctypes.c_size_t, _P]
_lib.moe_ep_expert_counts.restype = ctypes.c_int
_lib.moe_ep_expert_counts.argtypes = [_CFG, _P, _P, _P]
_lib.moe_ep_plan.restype = ctypes.c_int
_lib.moe_ep_plan.argtypes = [_CFG, ctypes.c_int32, ctypes.c_int32] + [_P] * 5 + [
    ctypes.c_int32, _P, _P]
_lib.moe_ep_dispatch_peer.restype = ctypes.c_int
_lib.moe_ep_dispatch_peer.argtypes = [_CFG, ctypes.c_int32, ctypes.c_int32] + [_P] * 9 + [
    ctypes.c_int32, _P]
_lib.moe_ep_combine_peer.restype = ctypes.c_int
_lib.moe_ep_combine_peer.argtypes = [_CFG, ctypes.c_int32, ctypes.c_int32] + [_P] * 8 + [
    ctypes.c_int32, _P]
_lib.moe_check_device_status.restype = ctypes.c_int
_lib.moe_check_device_status.argtypes = [_P, _P]


def lib() -> ctypes.CDLL:
    return _lib


def get_last_error() -> str:
    return _lib.moe_get_last_error().decode()


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoeError(st, where)


def workspace_size(cfg: MoeConfig) -> int:
    c = cfg.c()
    n = _lib.moe_workspace_size(ctypes.byref(c))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_workspace_size")
    return n


def workspace_offset(cfg: MoeConfig, item: str) -> int:
    c = cfg.c()
    off = _lib.moe_workspace_offset(ctypes.byref(c), WS_ITEMS[item])
    if off == ctypes.c_size_t(-1).value:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_workspace_offset")
    return off


def alloc_workspace(cfg: MoeConfig, device="cuda") -> torch.Tensor:
    """A zeroed workspace of moe_workspace_size bytes (256-byte aligned)."""
    return torch.zeros(workspace_size(cfg), dtype=torch.uint8, device=device)


def moe_route(cfg, x, w_router, bias, logits, topk_idx, topk_w, ws, stream=None):
    c = cfg.c()
    _check(_lib.moe_route(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(logits),
                          _ptr(topk_idx), _ptr(topk_w), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_route")


def moe_route_from_logits(cfg, logits, bias, topk_idx, topk_w, stream=None):
    c = cfg.c()
    _check(_lib.moe_route_from_logits(ctypes.byref(c), _ptr(logits), _ptr(bias), _ptr(topk_idx),
                                      _ptr(topk_w), _stream(stream)), "moe_route_from_logits")


def moe_bias_update(cfg, topk_idx, bias, gamma, stream=None):
    """noaux_tc expert-bias update in place: bias[e] += gamma * sign(mean load
    - load_e) over the batch's choices topk_idx [T, k]."""
    c = cfg.c()
    _check(_lib.moe_bias_update(ctypes.byref(c), _ptr(topk_idx), _ptr(bias), float(gamma),
                                _stream(stream)), "moe_bias_update")


def moe_permute(cfg, topk_idx, offsets, rows, pos, ws, stream=None):
    c = cfg.c()
    _check(_lib.moe_permute(ctypes.byref(c), _ptr(topk_idx), _ptr(offsets), _ptr(rows), _ptr(pos),
                            _ptr(ws), ws.numel(), _stream(stream)), "moe_permute")


def moe_permute_noalloc(cfg, topk_idx, offsets, rows, pos, stream=None):
    """moe_permute without a workspace, for callers that cannot allocate
    device memory; its scratch is a fixed array inside the library."""
    c = cfg.c()
    _check(_lib.moe_permute_noalloc(ctypes.byref(c), _ptr(topk_idx), _ptr(offsets), _ptr(rows),
                                    _ptr(pos), _stream(stream)), "moe_permute_noalloc")


def moe_expert_ffn(cfg, x, offsets, rows, pos, topk_w, w13, w2, w13s, w2s, y, y_shared, ws,
                   stream=None, w13_scale=None, w2_scale=None, w13s_scale=None, w2s_scale=None):
    c = cfg.c()
    _check(_lib.moe_expert_ffn(ctypes.byref(c), _ptr(x), _ptr(offsets), _ptr(rows), _ptr(pos),
                               _ptr(topk_w), _ptr(w13), _ptr(w13_scale), _ptr(w2), _ptr(w2_scale),
                               _ptr(w13s), _ptr(w13s_scale), _ptr(w2s), _ptr(w2s_scale), _ptr(y),
                               _ptr(y_shared), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_expert_ffn")


def moe_combine(cfg, y, pos, y_shared, out, stream=None):
    c = cfg.c()
    _check(_lib.moe_combine(ctypes.byref(c), _ptr(y), _ptr(pos), _ptr(y_shared), _ptr(out),
                            _stream(stream)), "moe_combine")


def moe_forward(cfg, x, w_router, bias, w13, w2, w13s, w2s, out, ws, stream=None,
                stage_events=None, w13_scale=None, w2_scale=None, w13s_scale=None,
                w2s_scale=None):
    """The whole layer.  stage_events: None or MOE_NUM_STAGES + 1 recorded
    torch.cuda.Event objects (enable_timing=True) to time the stages."""
    c = cfg.c()
    ev = None
    if stage_events is not None:
        assert len(stage_events) == MOE_NUM_STAGES + 1
        ev = (ctypes.c_void_p * (MOE_NUM_STAGES + 1))(*[e.cuda_event for e in stage_events])
    _check(_lib.moe_forward(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w13),
                            _ptr(w13_scale), _ptr(w2), _ptr(w2_scale), _ptr(w13s),
                            _ptr(w13s_scale), _ptr(w2s), _ptr(w2s_scale), _ptr(out), _ptr(ws),
                            ws.numel(), ev, _stream(stream)), "moe_forward")


def moe_rmsnorm(cfg, h, gamma, eps, u, stream=None):
    """Pre-norm of the block input: u = bf16(gamma * h / sqrt(mean(h^2) + eps))."""
    c = cfg.c()
    _check(_lib.moe_rmsnorm(ctypes.byref(c), _ptr(h), _ptr(gamma), float(eps), _ptr(u),
                            _stream(stream)), "moe_rmsnorm")


def moe_forward_block(cfg, h, gamma, eps, w_router, bias, w13, w2, w13s, w2s, out, ws,
                      stream=None, stage_events=None, w13_scale=None, w2_scale=None,
                      w13s_scale=None, w2s_scale=None):
    """One pre-norm block: out = h + MoE(RMSNorm(h)); out may be h."""
    c = cfg.c()
    ev = None
    if stage_events is not None:
        assert len(stage_events) == MOE_NUM_STAGES + 1
        ev = (ctypes.c_void_p * (MOE_NUM_STAGES + 1))(*[e.cuda_event for e in stage_events])
    _check(_lib.moe_forward_block(ctypes.byref(c), _ptr(h), _ptr(gamma), float(eps),
                                  _ptr(w_router), _ptr(bias), _ptr(w13), _ptr(w13_scale),
                                  _ptr(w2), _ptr(w2_scale), _ptr(w13s), _ptr(w13s_scale),
                                  _ptr(w2s), _ptr(w2s_scale), _ptr(out), _ptr(ws), ws.numel(),
                                  ev, _stream(stream)), "moe_forward_block")


def moe_quantize_act(x, q, scale, stream=None):
    """Step a0 of the FP8 layer: e4m3 codes and per-(row, 128-column) scales."""
    rows, cols = x.shape
    _check(_lib.moe_quantize_act(_ptr(x), rows, cols, _ptr(q), _ptr(scale), _stream(stream)),
           "moe_quantize_act")


def moe_ep_pack(cfg, ep_size, x, topk_idx, topk_w, offsets, pos, x_send, w_send, e_send,
                send_counts, stream=None):
    """Expert-parallel send buffer: routed rows in expert (= destination) order."""
    c = cfg.c()
    _check(_lib.moe_ep_pack(ctypes.byref(c), int(ep_size), _ptr(x), _ptr(topk_idx),
                            _ptr(topk_w), _ptr(offsets), _ptr(pos), _ptr(x_send), _ptr(w_send),
                            _ptr(e_send), _ptr(send_counts), _stream(stream)), "moe_ep_pack")


def moe_ep_expert_counts(cfg, offsets, counts, stream=None):
    c = cfg.c()
    _check(_lib.moe_ep_expert_counts(ctypes.byref(c), _ptr(offsets), _ptr(counts),
                                     _stream(stream)), "moe_ep_expert_counts")


def moe_ep_plan(cfg, ep_size, ep_rank, counts_all, exp_base, src_base, recv_offsets, recv_ident,
                recv_cap, ws, stream=None):
    c = cfg.c()
    _check(_lib.moe_ep_plan(ctypes.byref(c), int(ep_size), int(ep_rank), _ptr(counts_all),
                            _ptr(exp_base), _ptr(src_base), _ptr(recv_offsets), _ptr(recv_ident),
                            int(recv_cap), _ptr(ws), _stream(stream)), "moe_ep_plan")


def moe_ep_dispatch_peer(cfg, ep_size, ep_rank, x, topk_idx, topk_w, offsets, pos, exp_base,
                         src_base, x_recv_ptrs, w_recv_ptrs, recv_cap, stream=None):
    """x_recv_ptrs / w_recv_ptrs: int64 device tensors of the owners' buffer addresses."""
    c = cfg.c()
    _check(_lib.moe_ep_dispatch_peer(ctypes.byref(c), int(ep_size), int(ep_rank), _ptr(x),
                                     _ptr(topk_idx), _ptr(topk_w), _ptr(offsets), _ptr(pos),
                                     _ptr(exp_base), _ptr(src_base), _ptr(x_recv_ptrs),
                                     _ptr(w_recv_ptrs), int(recv_cap), _stream(stream)),
           "moe_ep_dispatch_peer")


def moe_ep_combine_peer(cfg, ep_size, ep_rank, topk_idx, offsets, pos, exp_base, src_base,
                        y_recv_ptrs, y_shared, out, recv_cap, stream=None):
    c = cfg.c()
    _check(_lib.moe_ep_combine_peer(ctypes.byref(c), int(ep_size), int(ep_rank), _ptr(topk_idx),
                                    _ptr(offsets), _ptr(pos), _ptr(exp_base), _ptr(src_base),
                                    _ptr(y_recv_ptrs), _ptr(y_shared), _ptr(out), int(recv_cap),
                                    _stream(stream)), "moe_ep_combine_peer")


def moe_shared_expert(cfg, x, w13s, w2s, y_shared, ws, stream=None):
    """The shared expert alone: y_shared (fp32) = SwiGLU_shared(x)."""
    c = cfg.c()
    _check(_lib.moe_shared_expert(ctypes.byref(c), _ptr(x), _ptr(w13s), _ptr(w2s),
                                  _ptr(y_shared), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_shared_expert")


def backward_workspace_size(cfg: MoeConfig) -> int:
    c = cfg.c()
    n = _lib.moe_backward_workspace_size(ctypes.byref(c))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_backward_workspace_size")
    return n


def alloc_backward_workspace(cfg: MoeConfig, device="cuda") -> torch.Tensor:
    """A workspace of moe_backward_workspace_size bytes (256-byte aligned)."""
    return torch.zeros(backward_workspace_size(cfg), dtype=torch.uint8, device=device)


def moe_backward(cfg, x, w_router, logits, topk_idx, topk_w, w13, w2, w13s, w2s, dout, dx,
                 dw_router, dw13, dw2, dw13s, dw2s, ws, dlogits=None, stream=None,
                 stage_events=None):
    """Gradients of sum(out * dout) with the forward's choice held fixed.
    stage_events: None or MOE_NUM_BWD_STAGES + 1 recorded torch.cuda.Event."""
    c = cfg.c()
    ev = None
    if stage_events is not None:
        assert len(stage_events) == MOE_NUM_BWD_STAGES + 1
        ev = (ctypes.c_void_p * (MOE_NUM_BWD_STAGES + 1))(*[e.cuda_event for e in stage_events])
    _check(_lib.moe_backward(ctypes.byref(c), _ptr(x), _ptr(w_router), _ptr(logits),
                             _ptr(topk_idx), _ptr(topk_w), _ptr(w13), _ptr(w2), _ptr(w13s),
                             _ptr(w2s), _ptr(dout), _ptr(dx), _ptr(dw_router), _ptr(dw13),
                             _ptr(dw2), _ptr(dw13s), _ptr(dw2s), _ptr(dlogits), _ptr(ws),
                             ws.numel(), ev, _stream(stream)), "moe_backward")


def moe_check_device_status(ws, stream=None):
    _check(_lib.moe_check_device_status(_ptr(ws), _stream(stream)), "moe_check_device_status")


def ws_view(ws: torch.Tensor, cfg: MoeConfig, item: str) -> torch.Tensor:
    """A typed view of an intermediate moe_forward leaves in the workspace."""
    off = workspace_offset(cfg, item)
    T, E, k, H = cfg.T, cfg.E, cfg.k, cfg.H
    shape, dt = {"logits": ((T, E), torch.float32), "topk_idx": ((T, k), torch.int32),
                 "topk_w": ((T, k), torch.float32), "offsets": ((E + 1,), torch.int32),
                 "rows": ((T * k,), torch.int32), "pos": ((T * k,), torch.int32),
                 "y": ((T * k, H), torch.float32 if k == 1 else torch.bfloat16),
                 "y_shared": ((T, H), torch.float32),
                 "u": ((T, H), torch.bfloat16)}[item]
    n = 1
    for d in shape:
        n *= d
    nbytes = n * torch.empty((), dtype=dt).element_size()
    return ws[off:off + nbytes].view(dt).view(shape)


# ---------------------------------------------------------------- DSA indexer (include/dsa.h)
@dataclass
class DsaConfig:
    """dsa_config_t: Sq queries, Sk keys, index heads of dim 128, top-k keys."""
    Sq: int
    Sk: int
    n_heads: int = 64
    head_dim: int = 128
    topk: int = 2048
    causal: bool = False
    q_offset: int = 0
    sorted: bool = True      # False: the same set by key index (no sort)

    def c(self) -> DsaConfigC:
        return DsaConfigC(self.Sq, self.Sk, self.n_heads, self.head_dim, self.topk,
                          int(bool(self.causal)), self.q_offset, int(bool(self.sorted)))


def dsa_workspace_size(cfg: DsaConfig) -> int:
    c = cfg.c()
    n = _lib.dsa_workspace_size(ctypes.byref(c))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "dsa_workspace_size")
    return n


def dsa_alloc_workspace(cfg: DsaConfig, device="cuda") -> torch.Tensor:
    return torch.zeros(dsa_workspace_size(cfg), dtype=torch.uint8, device=device)


def dsa_scores_view(ws: torch.Tensor, cfg: DsaConfig) -> torch.Tensor:
    off = _lib.dsa_workspace_scores_offset()
    return ws[off:off + cfg.Sq * cfg.Sk * 4].view(torch.float32).view(cfg.Sq, cfg.Sk)


def dsa_index_scores(cfg: DsaConfig, q, k, w, scores, ws, stream=None):
    c = cfg.c()
    _check(_lib.dsa_index_scores(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(w), _ptr(scores),
                                 _ptr(ws), ws.numel(), _stream(stream)), "dsa_index_scores")


def dsa_index_topk(cfg: DsaConfig, scores, idx, stream=None):
    c = cfg.c()
    _check(_lib.dsa_index_topk(ctypes.byref(c), _ptr(scores), _ptr(idx), _stream(stream)),
           "dsa_index_topk")


def dsa_indexer(cfg: DsaConfig, q, k, w, idx, ws, stream=None):
    c = cfg.c()
    _check(_lib.dsa_indexer(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(w), _ptr(idx), _ptr(ws),
                            ws.numel(), _stream(stream)), "dsa_indexer")
