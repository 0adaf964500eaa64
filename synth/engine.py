"""A synthetic workload on one GPU behind one msk handle: the seeded
weights and past KV filled on the device (synth.gpu), the handle and KV
cache created through the C ABI, and a step with the capture buffers set.
Used by the GPU tests, bench.py and the smoke check; it holds none of the
step's arithmetic (every step runs in libmsk.so's kernel)."""
import numpy as np
import torch

import synth.gpu as sg
import verify_step_megakernel_b200 as msk


def config_struct(w, max_seqs=None, max_tps=None, timeout_us=0, flags=0, tau=0):
    c = msk.Config()
    c.n_layers, c.d_model, c.n_q_heads, c.n_kv_heads = w.n_layers, w.d_model, w.n_q_heads, w.n_kv_heads
    c.head_dim, c.n_experts, c.top_k, c.expert_dim, c.window = (w.head_dim, w.n_experts, w.top_k, w.expert_dim,
                                                                 w.window)
    for i, s in enumerate(w.sliding):
        c.layer_is_sliding[i] = 1 if s else 0
    c.rms_eps = w.rms_eps
    c.max_seqs = max_seqs or w.n_seqs
    c.max_tokens_per_seq = max_tps or w.tokens_per_seq
    c.flags = flags
    c.wait_timeout_us = timeout_us
    c.expert_mma_min_tokens = tau
    return c


def layer_structs(wts):
    out = []
    for L in wts.layers:
        lw = msk.LayerWeights()
        lw.attn_norm_g, lw.q_norm_g, lw.k_norm_g = L["attn_norm_g"], L["q_norm_g"], L["k_norm_g"]
        lw.moe_norm_g, lw.router = L["moe_norm_g"], L["router"]
        for role in ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down"):
            c, s, gs = L[role]
            setattr(lw, role, msk.Nvfp4(c, s, gs))
        out.append(lw)
    return out


class Engine:
    """Weights + handle + KV cache of one workload on cuda:device."""

    def __init__(self, w, device=0, capacity=None, max_seqs=None, max_tps=None, timeout_us=0, flags=0,
                 past_per_seq=None, tau=0):
        self.w = w
        self.device = device
        self.dev = torch.device("cuda", device)
        self.wts = sg.DeviceWeights(w, device)
        self.cfg = config_struct(w, max_seqs, max_tps, timeout_us, flags, tau)
        self.h = msk.msk_create(self.cfg, layer_structs(self.wts), device)
        self.n_seqs = max_seqs or w.n_seqs
        self.past = past_per_seq or [w.past] * self.n_seqs
        cap = capacity or (max(self.past) + (max_tps or w.tokens_per_seq))
        self.kv = msk.msk_kv_create(self.h, self.n_seqs, cap)

    def fill_past(self, chunk=1 << 16):
        w = self.w
        hk = w.n_kv_heads * w.head_dim
        n0 = min(chunk, max(self.past) or 1)
        kb = torch.empty((n0, hk), dtype=torch.uint8, device=self.dev)
        vb = torch.empty((n0, hk), dtype=torch.uint8, device=self.dev)
        stream = torch.cuda.current_stream(self.dev).cuda_stream
        for l in range(w.n_layers):
            for b in range(self.n_seqs):
                for p0 in range(0, self.past[b], chunk):
                    n = min(chunk, self.past[b] - p0)
                    sg.past_chunk(w, l, b, p0, n, kb, vb, self.device)
                    msk.msk_kv_append(self.h, self.kv, l, b, p0, n, kb.data_ptr(), vb.data_ptr(), stream)
        torch.cuda.synchronize(self.dev)

    def step(self, hidden, positions, capture=True, stream=None, hold_barrier=0):
        """hidden: int16 [T][d] device tensor of bf16 bits; positions: int list [S][Tq].
        hold_barrier: the library's test hook (CTA 0 withholds its arrival at
        that grid barrier, so the step ends with a timeout)."""
        w = self.w
        pos = torch.tensor(positions, dtype=torch.int32, device=self.dev)
        S, Tq = pos.shape
        T = S * Tq
        out = torch.empty((T, w.d_model), dtype=torch.int16, device=self.dev)
        cap = {}
        if capture:
            L, k, E, qd = w.n_layers, w.top_k, w.n_experts, w.n_q_heads * w.head_dim
            kvd = w.n_kv_heads * w.head_dim
            cap = {"route_ids": torch.full((L, T, k), -1, dtype=torch.int16, device=self.dev),
                   "route_w": torch.zeros((L, T, k), dtype=torch.float32, device=self.dev),
                   "logits": torch.zeros((L, T, E), dtype=torch.float32, device=self.dev),
                   "attn_out": torch.zeros((L, T, qd), dtype=torch.float32, device=self.dev),
                   "k_pre": torch.zeros((L, T, kvd), dtype=torch.float32, device=self.dev),
                   "v_pre": torch.zeros((L, T, kvd), dtype=torch.float32, device=self.dev)}
            msk.msk_set_debug(self.h, cap["route_ids"].data_ptr(), cap["route_w"].data_ptr(),
                              cap["logits"].data_ptr(), cap["attn_out"].data_ptr(), k_pre=cap["k_pre"].data_ptr(),
                              v_pre=cap["v_pre"].data_ptr(), hold_barrier=hold_barrier)
        else:
            msk.msk_set_debug(self.h, hold_barrier=hold_barrier)
        st = stream if stream is not None else torch.cuda.current_stream(self.dev).cuda_stream
        msk.msk_step(self.h, hidden.data_ptr(), pos.data_ptr(), S, Tq, self.kv, out.data_ptr(), st)
        torch.cuda.synchronize(self.dev)
        status = msk.msk_step_status(self.h)
        res = {k_: v.cpu().numpy() for k_, v in cap.items()}
        res["hidden_out"] = out.cpu().numpy().view(np.uint16)
        res["status"] = status
        return res

    def read_kv(self, layer, seq, pos0, n):
        w = self.w
        k = np.zeros((n, w.n_kv_heads * w.head_dim), np.uint8)
        v = np.zeros_like(k)
        msk.msk_kv_read(self.h, self.kv, layer, seq, pos0, n, k.ctypes.data, v.ctypes.data)
        return k, v

    def close(self):
        if getattr(self, "kv", None):
            msk.msk_kv_destroy(self.kv)
            self.kv = None
        if getattr(self, "h", None):
            msk.msk_destroy(self.h)
            self.h = None
        self.wts = None
        if torch.cuda.is_available():
            torch.cuda.empty_cache()  # give the weights back for the next handle's own allocations

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


