"""Hand-built and small generated models for the oracle pins and GPU tests.

Hand-built models store weights whose values are exact e2m1 numbers with a
block scale of 1.0 and global scale 1, so every dequantised value is known
exactly; the expected results are then computed here with library routines
(numpy matmul, torch rms_norm/silu/softmax, torch's float8 conversion).
"""
import numpy as np
import torch

import synth
from synth.configs import Workload

E2M1 = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
E4M3_ONE = 0x38  # 1.0


def e2m1_code(v):
    c = E2M1[abs(float(v))]
    return c | (8 if v < 0 else 0)


def nvfp4_exact(W):
    """Encode a [rows][K] matrix of e2m1 values with block scale 1.0."""
    W = np.asarray(W, np.float64)
    rows, K = W.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    for r in range(rows):
        for k in range(0, K, 2):
            codes[r, k // 2] = e2m1_code(W[r, k]) | (e2m1_code(W[r, k + 1]) << 4)
    scales = np.full((rows, K // 16), E4M3_ONE, np.uint8)
    return codes, scales, 1.0


def e4m3_codes(x):
    """fp8 e4m3 codes of float values via torch (round to nearest even)."""
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e4m3_values(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)


def bf16_values(bits):
    return torch.from_numpy(np.asarray(bits, np.uint16).astype(np.int16)).view(torch.bfloat16).double().numpy()


def rmsnorm_ref(x, g, eps):
    x = torch.from_numpy(np.asarray(x, np.float64))
    return torch.nn.functional.rms_norm(x, (x.shape[-1],), torch.from_numpy(np.asarray(g, np.float64)),
                                        eps).numpy()


def hand_workload(**kw):
    base = dict(name="hand", n_layers=1, d_model=16, n_q_heads=1, n_kv_heads=1, head_dim=16,
                expert_dim=16, sliding=[0], n_seqs=1, tokens_per_seq=1, past=7, seed=1,
                n_experts=4, top_k=2, global_scale=False)
    base.update(kw)
    return Workload(**base)


class HandModel:
    """An ArraySource with explicit weights (dict of numpy arrays)."""

    def __init__(self, w, weights, past_k, past_v):
        self.w = w
        self.src = synth.ArraySource(w.n_layers, w.n_experts, w.n_seqs, w.n_kv_heads, w.head_dim)
        for l in range(w.n_layers):
            for name in ("attn_norm_g", "q_norm_g", "k_norm_g", "moe_norm_g", "router"):
                self.src.set_vec(l, name, weights[name])
            for role in ("wq", "wk", "wv", "wo"):
                self.src.set_nvfp4(l, role, 0, *nvfp4_exact(weights[role]))
            for e in range(w.n_experts):
                for role in ("w_gate", "w_up", "w_down"):
                    self.src.set_nvfp4(l, role, e, *nvfp4_exact(weights[role][e]))
            for b in range(w.n_seqs):
                for h in range(w.n_kv_heads):
                    self.src.set_past(l, b, h, past_k[l][b][h], past_v[l][b][h])


def generated_arrays(w):
    """All tensors of a small generated workload, as host arrays."""
    out = {"dense": {}, "experts": {}, "vec": {}}
    for l in range(w.n_layers):
        for role in ("wq", "wk", "wv", "wo"):
            out["dense"][(l, role)] = synth.host_nvfp4(w, role, l)
        for e in range(w.n_experts):
            for role in ("w_gate", "w_up", "w_down"):
                out["experts"][(l, role, e)] = synth.host_nvfp4(w, role, l, e)
        for name in ("attn_norm_g", "q_norm_g", "k_norm_g", "moe_norm_g", "router"):
            out["vec"][(l, name)] = synth.host_vec(w, name, l)
    return out


class ExtendableSource:
    """ArraySource over a generated workload whose past K/V can grow (used to
    replay a verify step as sequential decode steps)."""

    def __init__(self, w, arrays=None):
        self.w = w
        self.arrays = arrays or generated_arrays(w)
        self.past = {}
        for l in range(w.n_layers):
            for b in range(w.n_seqs):
                for h in range(w.n_kv_heads):
                    self.past[(l, b, h)] = synth.host_past(w, l, b, h, 0, w.past)
        self.rebuild()

    def append(self, l, b, h, k_row, v_row):
        k, v = self.past[(l, b, h)]
        self.past[(l, b, h)] = (np.vstack([k, k_row[None]]), np.vstack([v, v_row[None]]))

    def rebuild(self):
        w = self.w
        self.src = synth.ArraySource(w.n_layers, w.n_experts, w.n_seqs, w.n_kv_heads, w.head_dim)
        for (l, role), t in self.arrays["dense"].items():
            self.src.set_nvfp4(l, role, 0, *t)
        for (l, role, e), t in self.arrays["experts"].items():
            self.src.set_nvfp4(l, role, e, *t)
        for (l, name), v in self.arrays["vec"].items():
            self.src.set_vec(l, name, v)
        for (l, b, h), (k, v) in self.past.items():
            self.src.set_past(l, b, h, k, v)


def mini_workload(**kw):
    base = dict(name="mini", n_layers=2, d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16,
                expert_dim=32, sliding=[1, 0], n_seqs=2, tokens_per_seq=3, past=20, seed=77,
                n_experts=32, top_k=4, window=8)
    base.update(kw)
    return Workload(**base)
