"""Device-resident synthetic workloads: allocate with torch, fill on the GPU.

The fill kernels (synth_dev.cu) produce exactly the host generator's bytes,
so the oracle can regenerate any tensor on the host.
"""
import torch

from . import ROLES, dev_init, dev_nvfp4, dev_nvfp4_experts, dev_past, dev_vec, dev_hidden, nvfp4_shape

_inited = set()


def _init(device):
    if device not in _inited:
        with torch.cuda.device(device):
            dev_init()
        _inited.add(device)


class DeviceWeights:
    """All weights of a workload on one GPU.  layers[l] is a dict of
    pointers/global scales in the layout include/msk.h documents."""

    def __init__(self, w, device=0):
        _init(device)
        self.w = w
        self.device = device
        self.keep = []
        self.layers = []
        dev = torch.device("cuda", device)
        stream = torch.cuda.current_stream(dev).cuda_stream
        qd, kvd = w.n_q_heads * w.head_dim, w.n_kv_heads * w.head_dim
        self.bytes = 0
        keys = torch.empty(w.n_experts, dtype=torch.int64, device=dev)  # per-expert generator keys
        with torch.cuda.device(device):
            for l in range(w.n_layers):
                L = {}
                for name, n in (("attn_norm_g", w.d_model), ("q_norm_g", w.head_dim), ("k_norm_g", w.head_dim),
                                ("moe_norm_g", w.d_model), ("router", w.n_experts * w.d_model)):
                    t = torch.empty(n, dtype=torch.float32, device=dev)
                    dev_vec(w, name, l, t.data_ptr(), stream)
                    self.keep.append(t)
                    L[name] = t.data_ptr()
                for role in ("wq", "wk", "wv", "wo"):
                    rows, K = nvfp4_shape(w, role)
                    c = torch.empty(rows * K // 2, dtype=torch.uint8, device=dev)
                    s = torch.empty(rows * K // 16, dtype=torch.uint8, device=dev)
                    gs = dev_nvfp4(w, role, l, 0, c.data_ptr(), s.data_ptr(), stream)
                    self.keep += [c, s]
                    L[role] = (c.data_ptr(), s.data_ptr(), gs)
                    self.bytes += c.numel() + s.numel()
                for role in ("w_gate", "w_up", "w_down"):
                    rows, K = nvfp4_shape(w, role)
                    per_c, per_s = rows * K // 2, rows * K // 16
                    c = torch.empty(w.n_experts * per_c, dtype=torch.uint8, device=dev)
                    s = torch.empty(w.n_experts * per_s, dtype=torch.uint8, device=dev)
                    gs = dev_nvfp4_experts(w, role, l, keys.data_ptr(), c.data_ptr(), s.data_ptr(), stream)
                    self.keep += [c, s]
                    L[role] = (c.data_ptr(), s.data_ptr(), gs)
                    self.bytes += c.numel() + s.numel()
                self.layers.append(L)
        torch.cuda.synchronize(dev)


def hidden(w, device=0, n_seqs=None, tps=None, seq0=0):
    """bf16 hidden states [n_seqs*tps][d] on the GPU (as int16 storage)."""
    _init(device)
    n_seqs = w.n_seqs if n_seqs is None else n_seqs
    tps = w.tokens_per_seq if tps is None else tps
    dev = torch.device("cuda", device)
    out = torch.empty((n_seqs * tps, w.d_model), dtype=torch.int16, device=dev)
    keys = torch.empty(n_seqs * tps, dtype=torch.int64, device=dev)
    with torch.cuda.device(device):
        dev_hidden(w, seq0, n_seqs, tps, keys.data_ptr(), out.data_ptr(), torch.cuda.current_stream(dev).cuda_stream)
    return out


def past_chunk(w, layer, seq, pos0, n, k_buf, v_buf, device=0):
    """Fill k_buf/v_buf (uint8 [n][Hkv][hd] device tensors) with the past
    K/V codes of (layer, seq) for positions [pos0, pos0+n)."""
    _init(device)
    hd, H = w.head_dim, w.n_kv_heads
    stream = torch.cuda.current_stream(torch.device("cuda", device)).cuda_stream
    with torch.cuda.device(device):
        for h in range(H):
            dev_past(w, layer, seq, h, pos0, n, k_buf.data_ptr() + h * hd, v_buf.data_ptr() + h * hd, H * hd, stream)


__all__ = ["DeviceWeights", "hidden", "past_chunk", "ROLES"]
