"""Host-side validation of msk_create (include/msk.h): every shape rule and
argument check answers with its status code before any device call, so it
runs on CPU.  Weight pointers are aligned stand-ins that are never
dereferenced: the checks only test them for null and 16-byte alignment.

Each case is built so that only the rule under test can give the expected
answer: without a device a valid call ends with UNSUPPORTED, so a bad
argument (INVALID) is checked with otherwise valid weights, and an
unsupported shape (UNSUPPORTED) with a null router pointer, which the
weight checks after the shape rules would answer with INVALID."""
import math

import pytest
import torch

import synth
import verify_step_megakernel_b200 as msk
from synth.engine import config_struct

INVALID, UNSUPPORTED = 1, 2
FAKE = 0x10000  # aligned, never read


def _layers(n, **override):
    out = []
    for _ in range(n):
        lw = msk.LayerWeights()
        lw.attn_norm_g = lw.q_norm_g = lw.k_norm_g = lw.moe_norm_g = lw.router = FAKE
        for role in ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down"):
            setattr(lw, role, msk.Nvfp4(FAKE, FAKE, 1.0))
        for k, v in override.items():
            setattr(lw, k, v)
        out.append(lw)
    return out


def _code(cfg, layers):
    with pytest.raises(msk.MskError) as ei:
        msk.msk_create(cfg, layers, 0)
    return ei.value.code


def _cfg(**kw):
    w = synth.WORKLOADS["tiny"]
    c = config_struct(w)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


CASES = [
    ("no layers", dict(n_layers=0), INVALID),
    ("too many layers", dict(n_layers=65), INVALID),
    ("head dim 96", dict(head_dim=96), UNSUPPORTED),
    ("q heads not a multiple of kv heads", dict(n_q_heads=7, n_kv_heads=2), INVALID),
    ("d_model not a multiple of 256", dict(d_model=384), UNSUPPORTED),
    ("d_model above 4096", dict(d_model=8192), UNSUPPORTED),
    ("d_model above 512 not a multiple of 512", dict(d_model=768), UNSUPPORTED),
    ("q width 768", dict(n_q_heads=12), UNSUPPORTED),
    ("expert dim 96", dict(expert_dim=96), UNSUPPORTED),
    ("expert dim above 512 not a multiple of 512", dict(expert_dim=640), UNSUPPORTED),
    ("48 experts", dict(n_experts=48), UNSUPPORTED),
    ("512 experts", dict(n_experts=512), UNSUPPORTED),
    ("top_k 0", dict(top_k=0), INVALID),
    ("top_k 9", dict(top_k=9), INVALID),
    ("window 0", dict(window=0), INVALID),
    ("eps NaN", dict(rms_eps=math.nan), INVALID),
    ("eps negative", dict(rms_eps=-1e-6), INVALID),
    ("no sequences", dict(max_seqs=0), INVALID),
    ("more than 64 tokens", dict(max_seqs=16, max_tokens_per_seq=5), UNSUPPORTED),
    ("query rows per kv head above 64", dict(max_seqs=1, max_tokens_per_seq=9), UNSUPPORTED),
    ("negative wait limit", dict(wait_timeout_us=-1), INVALID),
    ("negative expert token threshold", dict(expert_mma_min_tokens=-1), INVALID),
]


@pytest.mark.parametrize("name,kw,code", CASES, ids=[c[0] for c in CASES])
def test_config_rule(name, kw, code):
    cfg = _cfg(**kw)
    n = max(1, min(cfg.n_layers, 64))
    layers = _layers(n) if code == INVALID else _layers(n, router=0)
    assert _code(cfg, layers) == code, name


@pytest.mark.parametrize("field,value", [
    ("router", 0), ("attn_norm_g", FAKE + 4), ("wq", msk.Nvfp4(0, FAKE, 1.0)),
    ("w_up", msk.Nvfp4(FAKE, FAKE + 8, 1.0)), ("w_down", msk.Nvfp4(FAKE, FAKE, 0.0)),
    ("wo", msk.Nvfp4(FAKE, FAKE, math.inf)),
], ids=["null router", "misaligned gain", "null codes", "misaligned scales", "zero global scale",
        "infinite global scale"])
def test_weight_pointer_checks(field, value):
    cfg = _cfg()
    assert _code(cfg, _layers(cfg.n_layers, **{field: value})) == INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the answer on a machine without a device")
def test_valid_config_without_a_device_is_unsupported():
    cfg = _cfg()
    assert _code(cfg, _layers(cfg.n_layers)) == UNSUPPORTED
