"""Pins of the oracle's indexing: NVFP4 blocks, scales and global scales,
the grouped-query head mapping, and the sliding-window edge.

Each case is built so that one plausible mistake in the oracle changes the
result beyond the test's tolerance:
- NVFP4 ("Expert Weight Quantization": e2m1 elements, one e4m3 scale per 16
  values, plus the fp32 per-tensor global scale of the format's second
  level): rows of four and two blocks with a different scale per block and
  per row and global scales 2^-5, 2^-3, 2^-6.  A block index of k/32, a
  scale taken from the wrong row, a swapped nibble order or a dropped or
  doubled global scale all move the expected values, which are computed
  here from the format tables (tests/golden/e2m1_values.txt, torch's
  float8_e4m3fn) and a numpy matmul.
- grouped-query attention (the pages' models share each kv head among a
  contiguous group of query heads; the reading is q head h -> kv head
  h / (Hq/Hkv)): 4 query heads over 2 kv heads whose keys and values
  differ, so h / 2 and h % 2 give different outputs, with closed forms
  (uniform attention -> the mean of V; one dominant key -> its V).
- the sliding window ("Model Architecture Details": 2,048-token window;
  the reading is keys j with pos - W < j <= pos): a dominant key exactly at
  pos - W + 1 must be attended, and the same key at pos - W must not be.
"""
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from tests._models import HandModel, bf16_bits, bf16_values, e4m3_codes, e4m3_values, hand_workload, rmsnorm_ref

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _e2m1_table():
    t = np.zeros(16)
    for line in open(os.path.join(GOLD, "e2m1_values.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            c, v = line.split()
            t[int(c)] = float(v)
    return t


E2M1 = _e2m1_table()
# normal e4m3 scale codes between 2^-3 and 2^3 (the block scales used below)
SCALE_CODES = np.array([c for c in range(0x18, 0x58)], np.uint8)


def _dequant(codes, scales, gs):
    """NVFP4 definition: value(r, c) = e2m1(nibble c of row r) x
    e4m3(scale[r][c // 16]) x global scale; nibble c is the low half of byte
    c // 2 when c is even."""
    rows, half = codes.shape
    K = 2 * half
    nib = np.empty((rows, K), np.int64)
    nib[:, 0::2] = codes & 0x0F
    nib[:, 1::2] = codes >> 4
    s = e4m3_values(scales)  # [rows][K/16]
    return E2M1[nib] * np.repeat(s, 16, axis=1) * gs


def _random_nvfp4(rng, rows, K, gs):
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    scales = rng.choice(SCALE_CODES, (rows, K // 16)).astype(np.uint8)
    return codes, scales, gs


class _Model:
    """HandModel with explicit NVFP4 tensors (codes, scales, global scale)
    for the roles given in `nv`; other weights as exact e2m1 matrices."""

    def __init__(self, w, dense, nv, past_k, past_v):
        self.src = HandModel(w, dense, past_k, past_v).src
        for (l, role, e), t in nv.items():
            self.src.set_nvfp4(l, role, e, *t)


def _zeros_model(w):
    d, qd, kvd, f, E = w.d_model, w.n_q_heads * w.head_dim, w.n_kv_heads * w.head_dim, w.expert_dim, w.n_experts
    return {
        "attn_norm_g": np.ones(d, np.float32), "moe_norm_g": np.ones(d, np.float32),
        "q_norm_g": np.ones(w.head_dim, np.float32), "k_norm_g": np.ones(w.head_dim, np.float32),
        "router": np.zeros((E, d), np.float32),
        "wq": np.zeros((qd, d)), "wk": np.zeros((kvd, d)), "wv": np.zeros((kvd, d)), "wo": np.zeros((d, qd)),
        "w_gate": [np.zeros((f, d))] * E, "w_up": [np.zeros((f, d))] * E, "w_down": [np.zeros((d, f))] * E,
    }


def _past(w, rng, P):
    kvd = w.n_kv_heads * w.head_dim
    pk = [[[e4m3_codes(rng.standard_normal((P, w.head_dim))) for _ in range(w.n_kv_heads)]]]
    pv = [[[e4m3_codes(rng.standard_normal((P, w.head_dim))) for _ in range(w.n_kv_heads)]]]
    assert kvd == w.n_kv_heads * w.head_dim
    return pk, pv


# ---- NVFP4 dequantisation: several blocks, per-block scales, global scale ---
def test_nvfp4_multiblock_dense_projection_with_global_scale():
    # d_model 64: every row of W_v holds four NVFP4 blocks, each with its own
    # scale; V before fp8 is x . deq(W_v)^T exactly (fp64)
    rng = np.random.default_rng(101)
    w = hand_workload(d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16, expert_dim=32, past=3)
    dense = _zeros_model(w)
    wv = _random_nvfp4(rng, 32, 64, 2.0 ** -5)
    pk, pv = _past(w, rng, w.past)
    m = _Model(w, dense, {(0, "wv", 0): wv}, pk, pv)
    h = bf16_bits(rng.standard_normal((1, 64)))
    o = oracle.step(w, m.src.ptr, h, w.positions(), threads=1)
    x = rmsnorm_ref(bf16_values(h), dense["attn_norm_g"], w.rms_eps)
    want = x @ _dequant(*wv).T
    assert np.allclose(o["v_pre"][0], want, rtol=1e-13, atol=1e-15)
    # the mistakes this rules out, each of which moves the result
    codes, scales, gs = wv
    wrong_block = E2M1[np.stack([codes & 15, codes >> 4], -1).reshape(32, 64)] * np.repeat(
        e4m3_values(scales)[:, :2], 32, axis=1) * gs  # block index k / 32
    wrong_row = _dequant(codes, scales[::-1].copy(), gs)  # scales of another row
    swapped = _dequant(((codes >> 4) | (codes << 4)).astype(np.uint8), scales, gs)  # nibble order
    for bad in (x @ wrong_block.T, x @ wrong_row.T, x @ swapped.T, x @ _dequant(codes, scales, 1.0).T,
                x @ _dequant(codes, scales, gs * gs).T):
        assert not np.allclose(o["v_pre"][0], bad, rtol=1e-3, atol=1e-6)


def test_nvfp4_multiblock_expert_with_global_scales():
    # one token routed to experts 1 and 3 with known weights; the experts'
    # gate/up rows hold four blocks (d 64) and the down rows two (f 32), every
    # block with its own scale, and each tensor its own global scale
    rng = np.random.default_rng(202)
    w = hand_workload(d_model=64, n_q_heads=4, n_kv_heads=1, head_dim=16, expert_dim=32, past=2)
    d, f = 64, 32
    dense = _zeros_model(w)
    router = np.zeros((4, d), np.float32)
    router[:, 0] = [0.5, 3.0, -1.0, 2.0]  # x2[0] > 0: experts 1 then 3
    dense["router"] = router
    nv = {}
    for e in range(4):
        nv[(0, "w_gate", e)] = _random_nvfp4(rng, f, d, 2.0 ** -5)
        nv[(0, "w_up", e)] = _random_nvfp4(rng, f, d, 2.0 ** -3)
        nv[(0, "w_down", e)] = _random_nvfp4(rng, d, f, 2.0 ** -6)
    pk, pv = _past(w, rng, w.past)
    m = _Model(w, dense, nv, pk, pv)
    hv = rng.standard_normal((1, d))
    hv[0, 0] = abs(hv[0, 0]) + 0.5
    h = bf16_bits(hv)
    o = oracle.step(w, m.src.ptr, h, w.positions(), threads=1)
    hin = bf16_values(h)[0]
    x2 = rmsnorm_ref(hin, dense["moe_norm_g"], w.rms_eps)
    logits = router.astype(np.float64) @ x2
    assert list(o["route_ids"][0, 0]) == [1, 3]
    wts = scipy.special.softmax(logits[[1, 3]])
    assert np.allclose(o["route_w"][0, 0], wts, rtol=1e-14)

    def expected(gs_down=None, gs_gate=None):
        out = hin.copy()
        for wt, e in zip(wts, (1, 3)):
            cg, sg_, gg = nv[(0, "w_gate", e)]
            cd, sd, gd = nv[(0, "w_down", e)]
            g = _dequant(cg, sg_, gg if gs_gate is None else gs_gate) @ x2
            u = _dequant(*nv[(0, "w_up", e)]) @ x2
            a = torch.nn.functional.silu(torch.from_numpy(g)).numpy() * u
            out += wt * (_dequant(cd, sd, gd if gs_down is None else gs_down) @ a)
        return out

    assert np.allclose(o["h_out"][0], expected(), rtol=1e-12, atol=1e-13)
    # a dropped global scale on the down or the gate projection moves it
    for bad in (expected(gs_down=1.0), expected(gs_gate=1.0), expected(gs_down=2.0 ** -12)):
        assert not np.allclose(o["h_out"][0], bad, rtol=1e-4, atol=1e-6)


# ---- grouped-query head mapping ---------------------------------------------
def _gqa_model(rng, P, dominant=None):
    w = hand_workload(d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16, expert_dim=32, past=P)
    dense = _zeros_model(w)
    pk, pv = _past(w, rng, P)
    if dominant is not None:
        # every query head along e0 (gain 3); kv head j has one key with
        # e0 = 8 at position dominant[j], every other key e0 = 0
        wq = np.zeros((64, 64))
        for hh in range(4):
            wq[hh * 16, :] = 1.0
        dense["wq"] = wq
        dense["q_norm_g"] = np.full(16, 3.0, np.float32)
        for j in range(2):
            kv = e4m3_values(pk[0][0][j]).copy()
            kv[:, 0] = 0.0
            kv[dominant[j], 0] = 8.0
            pk[0][0][j] = e4m3_codes(kv)
    return w, dense, pk, pv


def test_gqa_uniform_attention_uses_the_group_kv_head():
    # W_q = 0: every score is 0 and attention is the mean of V over the past
    # keys and this token's v (W_v = 0, so v = 0).  Past V of kv head j is
    # one constant row c_j: q heads 0, 1 see P/(P+1) c_0 and heads 2, 3 see
    # P/(P+1) c_1.
    rng = np.random.default_rng(303)
    P = 6
    w, dense, pk, pv = _gqa_model(rng, P)
    c = [e4m3_codes(rng.standard_normal(16)), e4m3_codes(rng.standard_normal(16))]
    for j in range(2):
        pv[0][0][j] = np.tile(c[j], (P, 1))
    m = HandModel(w, dense, pk, pv)
    h = bf16_bits(rng.standard_normal((1, 64)))
    o = oracle.step(w, m.src.ptr, h, w.positions(), threads=1)
    att = o["attn_out"][0, 0].reshape(4, 16)
    for hh in range(4):
        want = P / (P + 1) * e4m3_values(c[hh // 2])
        assert np.allclose(att[hh], want, rtol=1e-14, atol=1e-15), hh
    # h % Hkv would pair head 1 with kv head 1
    assert not np.allclose(att[1], P / (P + 1) * e4m3_values(c[1]), rtol=1e-3)


def test_gqa_dominant_key_comes_from_the_group_kv_head():
    # kv head 0's dominant key sits at position 2, kv head 1's at 5; a query
    # head attends (up to e^-24) to the dominant key of its group's kv head
    rng = np.random.default_rng(404)
    P = 9
    w, dense, pk, pv = _gqa_model(rng, P, dominant=(2, 5))
    m = HandModel(w, dense, pk, pv)
    h = bf16_bits(np.abs(rng.standard_normal((1, 64))) + 0.1)  # x[0] sum > 0 on every q head
    o = oracle.step(w, m.src.ptr, h, w.positions(), threads=1)
    att = o["attn_out"][0, 0].reshape(4, 16)
    V0, V1 = e4m3_values(pv[0][0][0]), e4m3_values(pv[0][0][1])
    for hh, want in ((0, V0[2]), (1, V0[2]), (2, V1[5]), (3, V1[5])):
        assert np.allclose(att[hh], want, rtol=0, atol=1e-8), hh
    assert not np.allclose(V0[2], V1[5], atol=1e-3)


# ---- sliding-window edge ------------------------------------------------------
def _window_case(key_pos, rng):
    # one sequence, P = 9 past keys, the new token at position 9, window 4:
    # keys 6, 7, 8, 9 are inside (9 - 4 < j <= 9)
    P, W = 9, 4
    w = hand_workload(past=P, sliding=[1], window=W)
    d = 16
    z = np.zeros((d, d))
    wq = np.zeros((d, d)); wq[0, :] = 1.0
    weights = {
        "attn_norm_g": np.ones(d, np.float32), "moe_norm_g": np.ones(d, np.float32),
        "q_norm_g": np.full(d, 3.0, np.float32), "k_norm_g": np.ones(d, np.float32),
        "router": np.zeros((4, d), np.float32),
        "wq": wq, "wk": z, "wv": np.eye(d), "wo": z,
        "w_gate": [z] * 4, "w_up": [z] * 4, "w_down": [z] * 4,
    }
    kv = rng.standard_normal((P, d))
    kv[:, 0] = 0.0
    kv[key_pos, 0] = 8.0
    pk = e4m3_codes(kv)
    pv = e4m3_codes(rng.standard_normal((P, d)))
    h = bf16_bits(np.abs(rng.standard_normal((1, d))) + 0.1)
    m = HandModel(w, weights, [[[pk]]], [[[pv]]])
    o = oracle.step(w, m.src.ptr, h, w.positions(), threads=1)
    return w, weights, h, pv, o


def test_window_first_key_is_attended():
    # the dominant key at pos - W + 1 = 6 is the window's oldest key: the
    # output is its V (up to e^-24)
    rng = np.random.default_rng(505)
    w, weights, h, pv, o = _window_case(6, rng)
    assert np.allclose(o["attn_out"][0, 0], e4m3_values(pv)[6], rtol=0, atol=1e-8)


def test_window_key_just_outside_is_not_attended():
    # the same key at pos - W = 5 lies outside: every key in the window
    # scores 0, so the output is the mean of V over keys 6, 7, 8 and this
    # token's own v (W_v = I)
    rng = np.random.default_rng(505)
    w, weights, h, pv, o = _window_case(5, rng)
    x = rmsnorm_ref(bf16_values(h), weights["attn_norm_g"], w.rms_eps)[0]
    V = np.vstack([e4m3_values(pv)[6:9], e4m3_values(e4m3_codes(x))[None]])
    assert np.allclose(o["attn_out"][0, 0], V.mean(0), rtol=1e-13, atol=1e-15)
    # a window one key wider would have taken the dominant key
    assert not np.allclose(o["attn_out"][0, 0], e4m3_values(pv)[5], atol=1e-2)
