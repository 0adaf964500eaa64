"""Seeded synthetic inputs for the decode/verify step (host and device).

Every tensor is a pure function of (seed, tensor stream, element index):
splitmix64 counters, a table-interpolated normal quantile, and the stored
formats' encoders (bf16 hidden, fp32 router, fp8-e4m3 past KV, NVFP4
weights).  The host fill (numpy arrays, the oracle's lazy source) and the
device fill (CUDA kernels writing into caller memory) are bit-identical.
This module holds none of the step's arithmetic.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build
from .configs import PROFILE_WORKLOADS, WORKLOADS, Workload  # noqa: F401

MAX_LAYERS = 64
ROLES = {"wq": 0, "wk": 1, "wv": 2, "wo": 3, "w_gate": 4, "w_up": 5, "w_down": 6}
VECS = {"attn_norm_g": 0, "q_norm_g": 1, "k_norm_g": 2, "moe_norm_g": 3, "router": 4}


class SyModel(C.Structure):
    _fields_ = [("seed", C.c_uint64),
                ("n_layers", C.c_int32), ("d_model", C.c_int32), ("n_q_heads", C.c_int32),
                ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("n_experts", C.c_int32),
                ("top_k", C.c_int32), ("expert_dim", C.c_int32), ("window", C.c_int32),
                ("is_sliding", C.c_uint8 * MAX_LAYERS), ("use_global_scale", C.c_int32)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        M = C.POINTER(SyModel)
        L.sy_fill_nvfp4.argtypes = [M, C.c_int, C.c_int, C.c_int, C.c_int64, C.c_int64, P, P]
        L.sy_fill_nvfp4.restype = C.c_float
        L.sy_fill_vec.argtypes = [M, C.c_int, C.c_int, P]
        L.sy_fill_hidden.argtypes = [M, C.c_int, C.c_int, P]
        L.sy_fill_past.argtypes = [M, C.c_int, C.c_int, C.c_int, C.c_int64, C.c_int64, P, P]
        L.sy_nvfp4_params.argtypes = [M, C.c_int, C.POINTER(C.c_float), C.POINTER(C.c_float)]
        L.sy_lazy_source_create.argtypes = [M]
        L.sy_lazy_source_create.restype = P
        L.sy_lazy_source_destroy.argtypes = [P]
        L.sy_lazy_source_bytes.argtypes = [P]
        L.sy_lazy_source_bytes.restype = C.c_int64
        L.sy_array_source_create.argtypes = [C.c_int] * 5
        L.sy_array_source_create.restype = P
        L.sy_array_source_destroy.argtypes = [P]
        L.sy_array_set_nvfp4.argtypes = [P, C.c_int, C.c_int, C.c_int, P, P, C.c_float]
        L.sy_array_set_vec.argtypes = [P, C.c_int, C.c_int, P]
        L.sy_array_set_past.argtypes = [P, C.c_int, C.c_int, C.c_int, P, P, C.c_int64]
        L.sy_set_threads.argtypes = [C.c_int]
        L.sy_table_copy.argtypes = [P]
        L.sy_table_bytes.restype = C.c_int
        L.sy_dev_init.restype = C.c_int
        L.sy_dev_fill_nvfp4.argtypes = [M, C.c_int, C.c_int, C.c_int, P, P, C.POINTER(C.c_float), P]
        L.sy_dev_fill_nvfp4.restype = C.c_int
        L.sy_dev_fill_nvfp4_experts.argtypes = [M, C.c_int, C.c_int, C.c_int, P, P, P, C.POINTER(C.c_float), P]
        L.sy_dev_fill_nvfp4_experts.restype = C.c_int
        L.sy_dev_fill_vec.argtypes = [M, C.c_int, C.c_int, P, P]
        L.sy_dev_fill_vec.restype = C.c_int
        L.sy_dev_fill_hidden.argtypes = [M, C.c_int, C.c_int, C.c_int, P, P, P]
        L.sy_dev_fill_hidden.restype = C.c_int
        L.sy_dev_fill_past.argtypes = [M, C.c_int, C.c_int, C.c_int, C.c_int64, C.c_int64, P, P, C.c_int64, P]
        L.sy_dev_fill_past.restype = C.c_int
        L.sy_set_threads(min(64, os.cpu_count() or 8))
        _lib = L
    return _lib


def model(w: "Workload") -> SyModel:
    m = SyModel()
    m.seed = w.seed
    m.n_layers, m.d_model, m.n_q_heads, m.n_kv_heads = w.n_layers, w.d_model, w.n_q_heads, w.n_kv_heads
    m.head_dim, m.n_experts, m.top_k, m.expert_dim = w.head_dim, w.n_experts, w.top_k, w.expert_dim
    m.window = w.window
    for i, s in enumerate(w.sliding):
        m.is_sliding[i] = 1 if s else 0
    m.use_global_scale = 1 if w.global_scale else 0
    return m


def nvfp4_shape(w, role):
    qd, kvd = w.n_q_heads * w.head_dim, w.n_kv_heads * w.head_dim
    return {"wq": (qd, w.d_model), "wk": (kvd, w.d_model), "wv": (kvd, w.d_model),
            "wo": (w.d_model, qd), "w_gate": (w.expert_dim, w.d_model),
            "w_up": (w.expert_dim, w.d_model), "w_down": (w.d_model, w.expert_dim)}[role]


def host_nvfp4(w, role, layer, expert=0, row0=0, nrows=None):
    """(codes [rows][K/2] u8, scales [rows][K/16] u8, global_scale) on the host."""
    rows, K = nvfp4_shape(w, role)
    nrows = rows - row0 if nrows is None else nrows
    codes = np.empty((nrows, K // 2), np.uint8)
    scales = np.empty((nrows, K // 16), np.uint8)
    m = model(w)
    gs = lib().sy_fill_nvfp4(C.byref(m), ROLES[role], layer, expert, row0, nrows,
                             codes.ctypes.data, scales.ctypes.data)
    return codes, scales, float(gs)


def host_vec(w, name, layer):
    n = {"q_norm_g": w.head_dim, "k_norm_g": w.head_dim,
         "router": w.n_experts * w.d_model}.get(name, w.d_model)
    out = np.empty(n, np.float32)
    m = model(w)
    lib().sy_fill_vec(C.byref(m), VECS[name], layer, out.ctypes.data)
    return out.reshape(w.n_experts, w.d_model) if name == "router" else out


def host_hidden(w, n_seqs=None, tps=None, seq0=0):
    """bf16 bits [n_seqs*tps][d]; row (s, t) is token t of sequence seq0+s."""
    n_seqs = w.n_seqs if n_seqs is None else n_seqs
    tps = w.tokens_per_seq if tps is None else tps
    out = np.empty((n_seqs * tps, w.d_model), np.uint16)
    m = model(w)
    for s in range(n_seqs):
        for t in range(tps):
            lib().sy_fill_hidden(C.byref(m), seq0 + s, t, out[s * tps + t].ctypes.data)
    return out


def host_past(w, layer, seq, head, pos0, n):
    k = np.empty((n, w.head_dim), np.uint8)
    v = np.empty((n, w.head_dim), np.uint8)
    m = model(w)
    lib().sy_fill_past(C.byref(m), layer, seq, head, pos0, n, k.ctypes.data, v.ctypes.data)
    return k, v


class LazySource:
    """msk_source regenerating any tensor on demand (cached)."""

    def __init__(self, w):
        self._m = model(w)
        self.ptr = lib().sy_lazy_source_create(C.byref(self._m))
        if not self.ptr:
            raise MemoryError("sy_lazy_source_create")

    def bytes(self):
        return lib().sy_lazy_source_bytes(self.ptr)

    def close(self):
        if self.ptr:
            lib().sy_lazy_source_destroy(self.ptr)
            self.ptr = None

    def __del__(self):
        self.close()


class ArraySource:
    """msk_source over host numpy arrays (kept alive here)."""

    def __init__(self, n_layers, n_experts, n_seqs, n_kv_heads, head_dim):
        self.ptr = lib().sy_array_source_create(n_layers, n_experts, n_seqs, n_kv_heads, head_dim)
        self._keep = []

    def set_nvfp4(self, layer, role, expert, codes, scales, gs):
        codes = np.ascontiguousarray(codes, np.uint8)
        scales = np.ascontiguousarray(scales, np.uint8)
        self._keep += [codes, scales]
        lib().sy_array_set_nvfp4(self.ptr, layer, ROLES[role], expert, codes.ctypes.data,
                                 scales.ctypes.data, float(gs))

    def set_vec(self, layer, name, v):
        v = np.ascontiguousarray(v, np.float32)
        self._keep.append(v)
        lib().sy_array_set_vec(self.ptr, layer, VECS[name], v.ctypes.data)

    def set_past(self, layer, seq, head, k, v):
        k = np.ascontiguousarray(k, np.uint8)
        v = np.ascontiguousarray(v, np.uint8)
        self._keep += [k, v]
        lib().sy_array_set_past(self.ptr, layer, seq, head, k.ctypes.data, v.ctypes.data, k.shape[0])

    def close(self):
        if self.ptr:
            lib().sy_array_source_destroy(self.ptr)
            self.ptr = None

    def __del__(self):
        self.close()


# ---- device fills (raw device pointers / stream handles as ints) ----------
def dev_init():
    rc = lib().sy_dev_init()
    if rc:
        raise RuntimeError(f"sy_dev_init failed: {rc}")


def dev_nvfp4(w, role, layer, expert, codes_ptr, scales_ptr, stream=0):
    gs = C.c_float()
    m = model(w)
    rc = lib().sy_dev_fill_nvfp4(C.byref(m), ROLES[role], layer, expert, codes_ptr, scales_ptr,
                                 C.byref(gs), stream)
    if rc:
        raise RuntimeError(f"sy_dev_fill_nvfp4: {rc}")
    return gs.value


def dev_nvfp4_experts(w, role, layer, keys_ptr, codes_ptr, scales_ptr, stream=0):
    """All n_experts tensors of an expert role in one launch; keys_ptr is
    device scratch of n_experts uint64."""
    gs = C.c_float()
    m = model(w)
    rc = lib().sy_dev_fill_nvfp4_experts(C.byref(m), ROLES[role], layer, w.n_experts, keys_ptr, codes_ptr,
                                         scales_ptr, C.byref(gs), stream)
    if rc:
        raise RuntimeError(f"sy_dev_fill_nvfp4_experts: {rc}")
    return gs.value


def dev_vec(w, name, layer, ptr, stream=0):
    m = model(w)
    rc = lib().sy_dev_fill_vec(C.byref(m), VECS[name], layer, ptr, stream)
    if rc:
        raise RuntimeError(f"sy_dev_fill_vec: {rc}")


def dev_hidden(w, seq0, n_seqs, tps, keys_ptr, out_ptr, stream=0):
    m = model(w)
    rc = lib().sy_dev_fill_hidden(C.byref(m), seq0, n_seqs, tps, keys_ptr, out_ptr, stream)
    if rc:
        raise RuntimeError(f"sy_dev_fill_hidden: {rc}")


def dev_past(w, layer, seq, head, pos0, n, k_ptr, v_ptr, row_stride, stream=0):
    """Past K/V of (layer, seq, head), positions [pos0, pos0+n), written at
    k_ptr + (pos - pos0) * row_stride (bytes), 16-byte aligned."""
    m = model(w)
    rc = lib().sy_dev_fill_past(C.byref(m), layer, seq, head, pos0, n, k_ptr, v_ptr, row_stride, stream)
    if rc:
        raise RuntimeError(f"sy_dev_fill_past: {rc}")
