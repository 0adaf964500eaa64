"""The step workloads: model shapes, batch shapes and KV lengths.

Shapes follow the scaled single-GPU stand-ins of the decoder the pages
describe ("Model Architecture Details": top-8 of 256 experts, sliding window
of 2,048 tokens mixed with full-context layers; "Expert Weight
Quantization": NVFP4 with one scale per 16 values; fp8 KV).  Value
distributions: NVFP4 weights from N(0, 1/fan_in); router fp32 N(0, 1/d);
RMSNorm and QK-norm gains U(0.8, 1.2); hidden states bf16 N(0, 1); past KV
fp8-e4m3 of N(0, 1).  Positions of sequence b are past, past+1, ...
"""
from dataclasses import dataclass, field, replace
from typing import List


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    expert_dim: int
    sliding: List[int]
    n_seqs: int
    tokens_per_seq: int
    past: int                 # past tokens per sequence already in the cache
    seed: int
    n_experts: int = 256
    top_k: int = 8
    window: int = 2048
    global_scale: bool = True  # per-tensor power-of-two NVFP4 global scale
    rms_eps: float = 1e-6
    extra: dict = field(default_factory=dict)

    @property
    def T(self):
        return self.n_seqs * self.tokens_per_seq

    def with_(self, **kw):
        return replace(self, **kw)

    def positions(self):
        """[n_seqs][tokens_per_seq] int positions."""
        return [[self.past + i for i in range(self.tokens_per_seq)] for _ in range(self.n_seqs)]


def _alt(n):
    return [1 if i % 2 == 0 else 0 for i in range(n)]


WORKLOADS = {
    # 2 layers (sliding, full), d=512, 8/1 heads, hd 64, f 128, 1 x 1 token, 4096 past
    "tiny": Workload("tiny", 2, 512, 8, 1, 64, 128, [1, 0], 1, 1, 4096, 0x5EED + 0),
    # 8 layers alternating sliding/full, d=2048, 16/2 heads, hd 128, f 512, 1 x 1, 32K past
    "dec8": Workload("dec8", 8, 2048, 16, 2, 128, 512, _alt(8), 1, 1, 32768, 0x5EED + 1),
    # same model as a verify step: 2 sequences x 8 draft tokens, 32K past each
    "ver8": Workload("ver8", 8, 2048, 16, 2, 128, 512, _alt(8), 2, 8, 32768, 0x5EED + 2),
    # 4 full layers, 1 x 4 tokens over 1,048,576 past tokens
    "long": Workload("long", 4, 2048, 16, 2, 128, 512, [0, 0, 0, 0], 1, 4, 1048576, 0x5EED + 3),
    # 16 layers (3 sliding : 1 full), d=4096, 32/4 heads, f 1024, 16 x 4 tokens, 128K past
    "large": Workload("large", 16, 4096, 32, 4, 128, 1024, [1, 1, 1, 0] * 4, 16, 4, 131072, 0x5EED + 4),
}
# profiling stand-in for the largest workload: its layer shapes and batch,
# two layers (sliding, full) and 8K past tokens, a few GB on the device
PROFILE_WORKLOADS = {
    "large2": Workload("large2", 2, 4096, 32, 4, 128, 1024, [1, 0], 16, 4, 8192, 0x5EED + 4),
}
