"""ctypes front end of the CPU oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the test suite, by the smoke check and
by the bench's CPU-baseline / reference arm.  The product library never
imports it.  Every function takes and returns numpy arrays; bf16 values travel
as their uint16 bit patterns, e4m3 values as uint8 codes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
          "-Wall", "-Wextra", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libmoe_oracle.so`` (gcc, no GPU)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("I", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
                ("group_topn", ctypes.c_int32), ("norm_topk_prob", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float), ("fp8", ctypes.c_int32)]


@dataclass
class Config:
    """Layer shape and routing options (names follow the Dots1 config fields)."""
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
    fp8: bool = False

    def c(self) -> _Cfg:
        return _Cfg(self.T, self.H, self.E, self.k, self.I, self.n_shared, self.n_group,
                    self.topk_group, self.group_topn, int(bool(self.norm_topk_prob)),
                    float(self.routed_scaling_factor), int(bool(self.fp8)))


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        _lib.orc_exp.restype = ctypes.c_float
        _lib.orc_exp.argtypes = [ctypes.c_float]
        _lib.orc_sigmoid.restype = ctypes.c_float
        _lib.orc_sigmoid.argtypes = [ctypes.c_float]
        _lib.orc_bf16_to_f32.restype = ctypes.c_float
        _lib.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        _lib.orc_f32_to_bf16.restype = ctypes.c_uint16
        _lib.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        _lib.orc_e4m3_to_f32.restype = ctypes.c_float
        _lib.orc_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        _lib.orc_f32_to_e4m3.restype = ctypes.c_uint8
        _lib.orc_f32_to_e4m3.argtypes = [ctypes.c_float]
        for name in ("orc_exp_n", "orc_sigmoid_n", "orc_e4m3_encode_n"):
            getattr(_lib, name).restype = None
            getattr(_lib, name).argtypes = [P, P, ctypes.c_int64]
        _lib.orc_router_logits.restype = None
        _lib.orc_router_logits.argtypes = [ctypes.POINTER(_Cfg), P, P, P]
        _lib.orc_route.restype = ctypes.c_int
        _lib.orc_route.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, P]
        _lib.orc_permute.restype = None
        _lib.orc_permute.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P]
        _lib.orc_quant_act_e4m3.restype = None
        _lib.orc_quant_act_e4m3.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P]
        _lib.orc_layer.restype = None
        _lib.orc_layer.argtypes = [ctypes.POINTER(_Cfg)] + [P] * 12 + [ctypes.c_int, P]
        _lib.orc_f64_to_bf16.restype = ctypes.c_uint16
        _lib.orc_f64_to_bf16.argtypes = [ctypes.c_double]
        _lib.orc_f64_to_bf16_n.restype = None
        _lib.orc_f64_to_bf16_n.argtypes = [P, P, ctypes.c_int64]
        _lib.orc_rmsnorm.restype = None
        _lib.orc_rmsnorm.argtypes = [ctypes.c_int, ctypes.c_int, P, P, ctypes.c_double, P, P]
        _lib.orc_dsa_scores.restype = None
        _lib.orc_dsa_scores.argtypes = [ctypes.c_int] * 4 + [P, P, P, ctypes.c_int, ctypes.c_int, P]
        _lib.orc_dsa_topk.restype = None
        _lib.orc_dsa_topk.argtypes = [ctypes.c_int] * 3 + [P, P]
        _lib.orc_set_threads.restype = ctypes.c_int
        _lib.orc_set_threads.argtypes = [ctypes.c_int]
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int = 0) -> int:
    """Set the OpenMP thread count (0 keeps the current one); returns it."""
    return lib().orc_set_threads(int(n))


def exp_f32(x) -> np.ndarray:
    x = _c(x, np.float32)
    y = np.empty_like(x)
    lib().orc_exp_n(_p(x), _p(y), x.size)
    return y


def sigmoid_f32(x) -> np.ndarray:
    x = _c(x, np.float32)
    y = np.empty_like(x)
    lib().orc_sigmoid_n(_p(x), _p(y), x.size)
    return y


def bf16_to_f32(b) -> np.ndarray:
    b = _c(b, np.uint16)
    return np.array([lib().orc_bf16_to_f32(int(v)) for v in b.ravel()],
                    dtype=np.float32).reshape(b.shape)


def f32_to_bf16(f) -> np.ndarray:
    f = _c(f, np.float32)
    return np.array([lib().orc_f32_to_bf16(float(v)) for v in f.ravel()],
                    dtype=np.uint16).reshape(f.shape)


def e4m3_to_f32(q) -> np.ndarray:
    q = _c(q, np.uint8)
    return np.array([lib().orc_e4m3_to_f32(int(v)) for v in q.ravel()],
                    dtype=np.float32).reshape(q.shape)


def f32_to_e4m3(f) -> np.ndarray:
    f = _c(f, np.float32)
    q = np.empty(f.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_n(_p(f), _p(q), f.size)
    return q


def quant_act_e4m3(v) -> tuple[np.ndarray, np.ndarray]:
    """Per-row, per-128-column e4m3 quantisation: returns (codes, scales)."""
    v = _c(v, np.float32)
    rows, cols = v.shape
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty((rows, (cols + 127) // 128), dtype=np.float32)
    lib().orc_quant_act_e4m3(rows, cols, _p(v), _p(q), _p(s))
    return q, s


def router_logits(cfg: Config, x_bf16, wg_bf16) -> np.ndarray:
    """fp64 logits [T, E] of bf16 x [T, H] against bf16 W_g [E, H]."""
    x = _c(x_bf16, np.uint16)
    wg = _c(wg_bf16, np.uint16)
    assert x.shape == (cfg.T, cfg.H) and wg.shape == (cfg.E, cfg.H)
    out = np.empty((cfg.T, cfg.E), dtype=np.float64)
    c = cfg.c()
    lib().orc_router_logits(ctypes.byref(c), _p(x), _p(wg), _p(out))
    return out


def route(cfg: Config, logits_f32, bias_f32):
    """(idx [T,k] int32, w [T,k] fp32, gap [T] fp32) from fp32 logits."""
    L = _c(logits_f32, np.float32)
    b = _c(bias_f32, np.float32)
    assert L.shape == (cfg.T, cfg.E) and b.shape == (cfg.E,)
    idx = np.empty((cfg.T, cfg.k), dtype=np.int32)
    w = np.empty((cfg.T, cfg.k), dtype=np.float32)
    gap = np.empty((cfg.T,), dtype=np.float32)
    c = cfg.c()
    rc = lib().orc_route(ctypes.byref(c), _p(L), _p(b), _p(idx), _p(w), _p(gap))
    if rc != 0:
        raise ValueError("oracle route: invalid configuration %r" % (cfg,))
    return idx, w, gap


def permute(cfg: Config, idx):
    """(offsets [E+1], rows [T*k], pos [T*k]) of the stable counting sort."""
    idx = _c(idx, np.int32)
    assert idx.shape == (cfg.T, cfg.k)
    offsets = np.empty((cfg.E + 1,), dtype=np.int32)
    rows = np.empty((cfg.T * cfg.k,), dtype=np.int32)
    pos = np.empty((cfg.T * cfg.k,), dtype=np.int32)
    c = cfg.c()
    lib().orc_permute(ctypes.byref(c), _p(idx), _p(offsets), _p(rows), _p(pos))
    return offsets, rows, pos


def layer(cfg: Config, x_bf16, idx, w, w13, w2, w13s, w2s, tokens=None,
          w13_scale=None, w2_scale=None, w13s_scale=None, w2s_scale=None) -> np.ndarray:
    """fp64 layer output [len(tokens), H] for the given routing.

    bf16 weights are uint16 arrays; fp8 weights (cfg.fp8) are uint8 codes with
    fp32 128x128 block scales.  Shapes: w13 [E, 2I, H], w2 [E, H, I],
    w13s [2*Is, H], w2s [H, Is] with Is = n_shared * I.
    """
    wdt = np.uint8 if cfg.fp8 else np.uint16
    x = _c(x_bf16, np.uint16)
    idx = _c(idx, np.int32)
    w = _c(w, np.float32)
    if tokens is None:
        tokens = np.arange(cfg.T, dtype=np.int32)
    tokens = _c(tokens, np.int32)
    Is = cfg.n_shared * cfg.I
    w13 = _c(w13, wdt)
    w2 = _c(w2, wdt)
    assert w13.size == cfg.E * 2 * cfg.I * cfg.H and w2.size == cfg.E * cfg.H * cfg.I
    w13s = _c(w13s, wdt) if Is > 0 else None
    w2s = _c(w2s, wdt) if Is > 0 else None
    if Is > 0:
        assert w13s.size == 2 * Is * cfg.H and w2s.size == cfg.H * Is
    sc = [_c(s, np.float32) for s in (w13_scale, w2_scale, w13s_scale, w2s_scale)]
    out = np.empty((tokens.size, cfg.H), dtype=np.float64)
    c = cfg.c()
    lib().orc_layer(ctypes.byref(c), _p(x), _p(idx), _p(w), _p(w13), _p(sc[0]), _p(w2),
                    _p(sc[1]), _p(w13s), _p(sc[2]), _p(w2s), _p(sc[3]), _p(tokens),
                    int(tokens.size), _p(out))
    return out


def f64_to_bf16(d) -> np.ndarray:
    """binary64 -> bf16 bits, round to nearest even in one step."""
    d = _c(d, np.float64)
    y = np.empty(d.shape, dtype=np.uint16)
    lib().orc_f64_to_bf16_n(_p(d), _p(y), d.size)
    return y


def rmsnorm(h_bf16, gamma_bf16, eps: float) -> tuple[np.ndarray, np.ndarray]:
    """Pre-norm of the layer input: (u bf16 bits [T, H], r = 1/sqrt(ms + eps) [T]).

    u = bf16(gamma * h / sqrt(mean(h^2) + eps)), evaluated in fp64, one rounding.
    """
    h = _c(h_bf16, np.uint16)
    g = _c(gamma_bf16, np.uint16)
    T, H = h.shape
    assert g.size == H
    u = np.empty((T, H), dtype=np.uint16)
    r = np.empty(T, dtype=np.float64)
    lib().orc_rmsnorm(T, H, _p(h), _p(g), float(eps), _p(u), _p(r))
    return u, r


def block(cfg: Config, h_bf16, gamma_bf16, eps: float, idx, w, w13, w2, w13s, w2s,
          tokens=None, **scales) -> np.ndarray:
    """fp64 output of one pre-norm block, h + layer(RMSNorm(h)), for the given
    routing (rows `tokens`)."""
    h = _c(h_bf16, np.uint16)
    u, _ = rmsnorm(h, gamma_bf16, eps)
    if tokens is None:
        tokens = np.arange(cfg.T, dtype=np.int32)
    tokens = _c(tokens, np.int32)
    moe = layer(cfg, u, idx, w, w13, w2, w13s, w2s, tokens=tokens, **scales)
    hv = (h[tokens].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return hv + moe


def dsa_scores(q_bf16, k_bf16, w_bf16, causal: bool = False, q_offset: int = 0) -> np.ndarray:
    """DSA indexer scores I[t, s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,h,:]) in fp64;
    q [Sq, nh, D], k [Sk, nh, D], w [Sq, nh] as bf16 bits.  Masked entries are -inf."""
    q = _c(q_bf16, np.uint16)
    k = _c(k_bf16, np.uint16)
    w = _c(w_bf16, np.uint16)
    Sq, nh, D = q.shape
    Sk = k.shape[0]
    assert k.shape == (Sk, nh, D) and w.shape == (Sq, nh)
    out = np.empty((Sq, Sk), dtype=np.float64)
    lib().orc_dsa_scores(Sq, Sk, nh, D, _p(q), _p(k), _p(w), int(bool(causal)), int(q_offset),
                         _p(out))
    return out


def dsa_topk(scores_f32, topk: int) -> np.ndarray:
    """Top-k keys per row of fp32 scores: score descending, equal scores by
    lower index, -inf never chosen, -1 padding."""
    sc = _c(scores_f32, np.float32)
    Sq, Sk = sc.shape
    idx = np.empty((Sq, topk), dtype=np.int32)
    lib().orc_dsa_topk(Sq, Sk, int(topk), _p(sc), _p(idx))
    return idx
