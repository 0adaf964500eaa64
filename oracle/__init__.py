"""TEST INFRASTRUCTURE: ctypes front end of the fp64 CPU oracle.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
reference leg may import this package.  The product path never does.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

MAX_LAYERS = 64


class OrCfg(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("d_model", C.c_int32), ("n_q_heads", C.c_int32),
                ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("n_experts", C.c_int32),
                ("top_k", C.c_int32), ("expert_dim", C.c_int32), ("window", C.c_int32),
                ("is_sliding", C.c_uint8 * MAX_LAYERS), ("rms_eps", C.c_double)]


class OrOut(C.Structure):
    _fields_ = [("hidden_out", C.c_void_p), ("h_out", C.c_void_p), ("route_ids", C.c_void_p),
                ("route_w", C.c_void_p), ("route_gap", C.c_void_p), ("logits", C.c_void_p),
                ("attn_out", C.c_void_p), ("k_new", C.c_void_p), ("v_new", C.c_void_p),
                ("s_max_minus_bound", C.c_void_p), ("n_distinct", C.c_void_p), ("k_pre", C.c_void_p),
                ("v_pre", C.c_void_p)]


class OrForce(C.Structure):
    _fields_ = [("ids", C.c_void_p), ("k", C.c_void_p), ("v", C.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(_build.build())
        P = C.c_void_p
        L.msk_oracle_step.argtypes = [C.POINTER(OrCfg), P, C.c_int, C.c_int, P, P, P, C.POINTER(OrForce),
                                      C.c_int, C.POINTER(OrOut)]
        L.msk_oracle_step.restype = C.c_int
        L.msk_or_e2m1_decode.argtypes = [C.c_int]
        L.msk_or_e2m1_decode.restype = C.c_double
        L.msk_or_e4m3_decode.argtypes = [C.c_int]
        L.msk_or_e4m3_decode.restype = C.c_double
        L.msk_or_e4m3_encode.argtypes = [C.c_double]
        L.msk_or_e4m3_encode.restype = C.c_int
        L.msk_or_e4m3_encode_n.argtypes = [P, C.c_int64, P]
        L.msk_or_e4m3_encode_n.restype = None
        L.msk_or_bf16_encode.argtypes = [C.c_double]
        L.msk_or_bf16_encode.restype = C.c_uint16
        L.msk_or_bf16_decode.argtypes = [C.c_uint16]
        L.msk_or_bf16_decode.restype = C.c_double
        L.msk_or_rmsnorm.argtypes = [P, P, C.c_int, C.c_double, P]
        L.msk_or_silu.argtypes = [C.c_double]
        L.msk_or_silu.restype = C.c_double
        L.msk_or_topk.argtypes = [P, C.c_int, C.c_int, P, P, P]
        L.msk_or_route_weights.argtypes = [P, P, C.c_int, P]
        L.msk_or_attend.argtypes = [P, P, P, C.c_int64, C.c_int, C.c_double, P, P]
        _lib = L
    return _lib


def cfg_struct(w):
    c = OrCfg()
    c.n_layers, c.d_model, c.n_q_heads, c.n_kv_heads = w.n_layers, w.d_model, w.n_q_heads, w.n_kv_heads
    c.head_dim, c.n_experts, c.top_k, c.expert_dim, c.window = (w.head_dim, w.n_experts, w.top_k,
                                                                 w.expert_dim, w.window)
    for i, s in enumerate(w.sliding):
        c.is_sliding[i] = 1 if s else 0
    c.rms_eps = w.rms_eps
    return c


def step(w, source_ptr, hidden_in, positions, seq_ids=None, forced_ids=None, forced_k=None, forced_v=None,
         threads=None):
    """Run one oracle step.  hidden_in: uint16 [T][d] bf16 bits; positions:
    int [n_seqs][tps]; forced_*: optional replacements (-1 = oracle's own
    decision) of near-tied routing [L][T][k] and of fp8 KV codes at rounding
    midpoints [L][T][Hkv*hd].  Returns a dict of numpy outputs."""
    positions = np.ascontiguousarray(positions, np.int32)
    n_seqs, tps = positions.shape
    T = n_seqs * tps
    L, d, E, k = w.n_layers, w.d_model, w.n_experts, w.top_k
    qd, kvd = w.n_q_heads * w.head_dim, w.n_kv_heads * w.head_dim
    hidden_in = np.ascontiguousarray(hidden_in, np.uint16).reshape(T, d)
    o = {
        "hidden_out": np.zeros((T, d), np.uint16), "h_out": np.zeros((T, d)),
        "route_ids": np.zeros((L, T, k), np.int16), "route_w": np.zeros((L, T, k)),
        "route_gap": np.zeros((L, T)), "logits": np.zeros((L, T, E)),
        "attn_out": np.zeros((L, T, qd)), "k_new": np.zeros((L, T, kvd), np.uint8),
        "v_new": np.zeros((L, T, kvd), np.uint8), "s_max_minus_bound": np.zeros(L),
        "n_distinct": np.zeros(L, np.int32), "k_pre": np.zeros((L, T, kvd)), "v_pre": np.zeros((L, T, kvd)),
    }
    out = OrOut(*[o[f].ctypes.data for f, _ in OrOut._fields_])
    sid = None if seq_ids is None else np.ascontiguousarray(seq_ids, np.int32)
    fr = None if forced_ids is None else np.ascontiguousarray(forced_ids, np.int16).reshape(L, T, k)
    fk = None if forced_k is None else np.ascontiguousarray(forced_k, np.int16).reshape(L, T, kvd)
    fv = None if forced_v is None else np.ascontiguousarray(forced_v, np.int16).reshape(L, T, kvd)
    force = OrForce(None if fr is None else fr.ctypes.data, None if fk is None else fk.ctypes.data,
                    None if fv is None else fv.ctypes.data)
    cfg = cfg_struct(w)
    nt = threads if threads else min(64, os.cpu_count() or 1)
    rc = lib().msk_oracle_step(C.byref(cfg), source_ptr, n_seqs, tps,
                               None if sid is None else sid.ctypes.data, positions.ctypes.data,
                               hidden_in.ctypes.data, C.byref(force), nt, C.byref(out))
    if rc:
        raise RuntimeError(f"msk_oracle_step failed: {rc}")
    return o


def topk(logits, k):
    logits = np.ascontiguousarray(logits, np.float64)
    ids = np.zeros(k, np.int16)
    w = np.zeros(k)
    gap = C.c_double()
    lib().msk_or_topk(logits.ctypes.data, len(logits), k, ids.ctypes.data, w.ctypes.data, C.byref(gap))
    return ids, w, gap.value


def attend(q, K, V, scale):
    q = np.ascontiguousarray(q, np.float64)
    K = np.ascontiguousarray(K, np.float64)
    V = np.ascontiguousarray(V, np.float64)
    o = np.zeros(q.shape[0])
    smax = C.c_double()
    lib().msk_or_attend(q.ctypes.data, K.ctypes.data, V.ctypes.data, K.shape[0], q.shape[0], scale,
                        o.ctypes.data, C.byref(smax))
    return o, smax.value


def e4m3_encode(x):
    """The oracle's fp8 e4m3 encoder (nearest even, saturating) over an array."""
    x = np.ascontiguousarray(x, np.float64)
    out = np.zeros(x.shape, np.uint8)
    lib().msk_or_e4m3_encode_n(x.ctypes.data, x.size, out.ctypes.data)
    return out


def rmsnorm(x, g, eps):
    x = np.ascontiguousarray(x, np.float64)
    g = np.ascontiguousarray(g, np.float32)
    y = np.zeros_like(x)
    lib().msk_or_rmsnorm(x.ctypes.data, g.ctypes.data, len(x), eps, y.ctypes.data)
    return y
