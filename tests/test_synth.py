"""The seeded input recipe: distributions and determinism (host side).

The device fill is checked bit-for-bit against this host fill in
test_gpu_synth.py.
"""
import numpy as np
import pytest
import scipy.stats

import synth
from tests._models import bf16_values, e4m3_values, mini_workload


def test_hidden_is_standard_normal_bf16():
    w = synth.WORKLOADS["large"].with_(n_seqs=16, tokens_per_seq=16)
    x = bf16_values(synth.host_hidden(w)).ravel()
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    qs = [0.001, 0.025, 0.16, 0.5, 0.84, 0.975, 0.999]
    assert np.allclose(np.quantile(x, qs), scipy.stats.norm.ppf(qs), atol=0.03)
    # tails of the table-interpolated quantile reach ~6.3 sigma at most
    assert np.abs(x).max() < 6.5


def test_past_kv_is_fp8_of_standard_normal():
    w = synth.WORKLOADS["dec8"]
    k, v = synth.host_past(w, 3, 0, 1, 1000, 4096)
    kv = e4m3_values(k).ravel()
    assert abs(kv.mean()) < 0.01 and abs(kv.std() - 1) < 0.01
    assert k.shape == (4096, 128) and not np.array_equal(k, v)
    k2, _ = synth.host_past(w, 3, 0, 1, 1000 + 17, 10)
    assert np.array_equal(k2, k[17:27])  # any range regenerates identically


def test_nvfp4_weights_scale_and_spread():
    w = synth.WORKLOADS["dec8"]
    codes, scales, gs = synth.host_nvfp4(w, "w_gate", 2, 17)
    assert codes.shape == (512, 1024) and scales.shape == (512, 128)
    sigma = 1 / np.sqrt(2048)
    assert gs == 2.0 ** np.ceil(np.log2(8 * sigma / 6 / 448))
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6])
    lo, hi = grid[codes & 15], grid[codes >> 4]
    vals = np.stack([lo, hi], -1).reshape(512, 2048)
    deq = vals * np.repeat(e4m3_values(scales), 16, axis=1) * gs
    assert abs(deq.std() / sigma - 1) < 0.03
    # each block's largest |code| is 6 unless the scale rounded up (then 4)
    bmax = np.abs(vals).reshape(512, 128, 16).max(-1)
    assert np.isin(bmax, [3.0, 4.0, 6.0]).all() and (bmax == 6.0).mean() > 0.4


def test_fills_are_deterministic_and_keyed():
    w = synth.WORKLOADS["tiny"]
    a = synth.host_nvfp4(w, "wq", 0)
    b = synth.host_nvfp4(w, "wq", 0)
    c = synth.host_nvfp4(w, "wq", 1)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert not np.array_equal(a[0], c[0])
    part = synth.host_nvfp4(w, "wq", 0, row0=64, nrows=32)
    assert np.array_equal(part[0], a[0][64:96]) and np.array_equal(part[1], a[1][64:96])
    g = synth.host_vec(w, "q_norm_g", 1)
    assert g.min() >= 0.8 and g.max() < 1.2
    r = synth.host_vec(w, "router", 0)
    assert r.shape == (256, 512) and abs(r.std() * np.sqrt(512) - 1) < 0.02


def test_lazy_source_counts_bytes():
    w = mini_workload()
    src = synth.LazySource(w)
    assert src.bytes() == 0
    src.close()
