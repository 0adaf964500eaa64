"""Python binding of libmsk.so (include/msk.h): argument marshalling only.

Every step of the decode/verify path runs in the library's CUDA kernel; this
module converts Python values to the C structs and raises on error codes.
Pointers are plain integers (e.g. torch.Tensor.data_ptr()).  Importing
fails loudly when the library cannot be built or loaded: there is no CPU
fallback.
"""
import ctypes as C
import os

from . import _build

MAX_LAYERS = 64
MAX_TOKENS = 64

STATUS = {0: "MSK_OK", 1: "MSK_ERR_INVALID_ARG", 2: "MSK_ERR_UNSUPPORTED", 3: "MSK_ERR_OOM", 4: "MSK_ERR_CUDA",
          5: "MSK_ERR_BOUND", 6: "MSK_ERR_KV_RANGE", 7: "MSK_ERR_TIMEOUT", 8: "MSK_ERR_DEVICE"}
F_TRACE = 1
F_TC_EXPERTS = 2  # gate/up on the block-scaled tensor cores
TAU_DEFAULT = 1  # expert_mma_min_tokens when 0 is passed
TAU_NEVER = 0x7FFFFFFF  # every unit's gate/up on the CUDA-core path


class MskError(RuntimeError):
    def __init__(self, code, what):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


class Nvfp4(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("global_scale", C.c_float)]


class Config(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("d_model", C.c_int32), ("n_q_heads", C.c_int32),
                ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("n_experts", C.c_int32),
                ("top_k", C.c_int32), ("expert_dim", C.c_int32), ("window", C.c_int32),
                ("layer_is_sliding", C.c_uint8 * MAX_LAYERS), ("rms_eps", C.c_float),
                ("max_seqs", C.c_int32), ("max_tokens_per_seq", C.c_int32), ("flags", C.c_uint32),
                ("wait_timeout_us", C.c_int32), ("expert_mma_min_tokens", C.c_int32)]


class LayerWeights(C.Structure):
    _fields_ = [("attn_norm_g", C.c_void_p), ("q_norm_g", C.c_void_p), ("k_norm_g", C.c_void_p),
                ("moe_norm_g", C.c_void_p), ("router", C.c_void_p),
                ("wq", Nvfp4), ("wk", Nvfp4), ("wv", Nvfp4), ("wo", Nvfp4),
                ("w_gate", Nvfp4), ("w_up", Nvfp4), ("w_down", Nvfp4)]


class Debug(C.Structure):
    _fields_ = [("route_ids", C.c_void_p), ("route_w", C.c_void_p), ("logits", C.c_void_p),
                ("attn_out", C.c_void_p), ("trace", C.c_void_p), ("k_pre", C.c_void_p), ("v_pre", C.c_void_p),
                ("hold_barrier", C.c_int32)]


class Stats(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("n_distinct", C.c_int32 * MAX_LAYERS),
                ("algorithmic_bytes", C.c_int64), ("weight_bytes", C.c_int64), ("kv_bytes", C.c_int64),
                ("scratch_bytes", C.c_int64), ("repacked_bytes", C.c_int64)]


_lib = None
EXPORTS = ["msk_create", "msk_destroy", "msk_kv_create", "msk_kv_destroy", "msk_kv_append", "msk_kv_encode",
           "msk_kv_read", "msk_step", "msk_step_static", "msk_step_status", "msk_step_status_at", "msk_set_debug",
           "msk_query", "msk_status_string"]
STATIC_SCRATCH_BYTES = 8 << 20


def lib():
    """Load (building first if the sources changed) libmsk.so."""
    global _lib
    if _lib is None:
        path = _build.LIB if os.environ.get("MSK_NO_BUILD") else _build.build()
        L = C.CDLL(path)
        P, I, I64 = C.c_void_p, C.c_int, C.c_int64
        L.msk_create.argtypes = [C.POINTER(Config), C.POINTER(LayerWeights), I, C.POINTER(P)]
        L.msk_destroy.argtypes = [P]
        L.msk_destroy.restype = None
        L.msk_kv_create.argtypes = [P, I, I64, C.POINTER(P)]
        L.msk_kv_destroy.argtypes = [P]
        L.msk_kv_destroy.restype = None
        L.msk_kv_append.argtypes = [P, P, I, I, I64, I64, P, P, P]
        L.msk_kv_read.argtypes = [P, P, I, I, I64, I64, P, P]
        L.msk_kv_encode.argtypes = [P, P, I64, P]
        L.msk_step.argtypes = [P, P, P, I, I, P, P, P]
        L.msk_step_static.argtypes = [P, P, P, I, I, P, P, P]
        L.msk_step_status.argtypes = [P]
        L.msk_step_status_at.argtypes = [P, C.POINTER(C.c_int32), C.POINTER(C.c_int32), C.POINTER(C.c_int32)]
        L.msk_set_debug.argtypes = [P, C.POINTER(Debug)]
        L.msk_query.argtypes = [P, C.POINTER(Stats)]
        L.msk_status_string.argtypes = [I]
        L.msk_status_string.restype = C.c_char_p
        for name in ("msk_create", "msk_kv_create", "msk_kv_append", "msk_kv_encode", "msk_kv_read", "msk_step",
                     "msk_step_static", "msk_step_status", "msk_step_status_at", "msk_set_debug", "msk_query"):
            getattr(L, name).restype = C.c_int
        _lib = L
    return _lib


def _check(rc, what):
    if rc != 0:
        raise MskError(rc, what)


def msk_create(config: Config, layers, device: int = 0) -> int:
    arr = (LayerWeights * len(layers))(*layers)
    h = C.c_void_p()
    _check(lib().msk_create(C.byref(config), arr, device, C.byref(h)), "msk_create")
    return h.value


def msk_destroy(h: int) -> None:
    lib().msk_destroy(h)


def msk_kv_create(h: int, n_seqs: int, capacity: int) -> int:
    kv = C.c_void_p()
    _check(lib().msk_kv_create(h, n_seqs, capacity, C.byref(kv)), "msk_kv_create")
    return kv.value


def msk_kv_destroy(kv: int) -> None:
    lib().msk_kv_destroy(kv)


def msk_kv_append(h, kv, layer, seq, pos0, n, k_fp8, v_fp8, stream=0):
    _check(lib().msk_kv_append(h, kv, layer, seq, pos0, n, k_fp8, v_fp8, stream), "msk_kv_append")


def msk_kv_encode(in_f32, out_u8, n, stream=0):
    _check(lib().msk_kv_encode(in_f32, out_u8, n, stream), "msk_kv_encode")


def msk_kv_read(h, kv, layer, seq, pos0, n, k_out, v_out):
    _check(lib().msk_kv_read(h, kv, layer, seq, pos0, n, k_out, v_out), "msk_kv_read")


def msk_step(h, hidden_in, positions, n_seqs, tokens_per_seq, kv, hidden_out, stream=0):
    _check(lib().msk_step(h, hidden_in, positions, n_seqs, tokens_per_seq, kv, hidden_out, stream), "msk_step")


def msk_step_static(h, hidden_in, positions, n_seqs, tokens_per_seq, kv, hidden_out, stream=0):
    """msk_step with its working memory in the library's fixed array (no
    allocation); see include/msk.h for who needs it and its limits."""
    _check(lib().msk_step_static(h, hidden_in, positions, n_seqs, tokens_per_seq, kv, hidden_out, stream),
           "msk_step_static")


def msk_step_status(h) -> int:
    return lib().msk_step_status(h)


def msk_step_status_at(h):
    """(status, layer, phase, cta) of the steps since the last status call."""
    a, b, c = C.c_int32(), C.c_int32(), C.c_int32()
    st = lib().msk_step_status_at(h, C.byref(a), C.byref(b), C.byref(c))
    return st, a.value, b.value, c.value


def msk_set_debug(h, route_ids=0, route_w=0, logits=0, attn_out=0, trace=0, k_pre=0, v_pre=0, hold_barrier=0):
    d = Debug(route_ids or None, route_w or None, logits or None, attn_out or None, trace or None, k_pre or None,
              v_pre or None, int(hold_barrier))
    _check(lib().msk_set_debug(h, C.byref(d)), "msk_set_debug")


def msk_query(h) -> Stats:
    s = Stats()
    _check(lib().msk_query(h, C.byref(s)), "msk_query")
    return s


def msk_status_string(code: int) -> str:
    return lib().msk_status_string(code).decode()
