"""Pins of the fp64 oracle against closed forms, brute force, library
routines and invariants of the step.

- fixed-bound softmax ("Removing Attention Bottlenecks": QK-norm bounds the
  scores, so no running max is needed) equals max-subtracted softmax;
- top-k routing ("8 of 256 experts") equals a brute-force full sort with
  (logit desc, index asc), weights equal the library softmax of the k;
- RMSNorm and SiLU equal torch's routines; constant rows give g * sign;
- hand-computable one-layer / four-expert cases with exact weights;
- a verify step of T tokens equals T sequential decode steps; a sliding
  window longer than the context equals full attention; sequences in a batch
  are independent.
"""
import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth
from tests._models import (ExtendableSource, HandModel, bf16_bits, bf16_values, e4m3_codes, e4m3_values,
                           hand_workload, mini_workload, rmsnorm_ref)


# ---- building blocks --------------------------------------------------------
@pytest.mark.parametrize("spread", [0.5, 4.0, 16.0, 39.0])
def test_fixed_bound_softmax_equals_max_subtracted(spread):
    rng = np.random.default_rng(int(spread * 10))
    hd, n = 64, 300
    q = rng.standard_normal(hd)
    q *= np.sqrt(hd) / np.linalg.norm(q)
    K = rng.standard_normal((n, hd))
    K *= (np.sqrt(hd) / np.linalg.norm(K, axis=1))[:, None]
    V = rng.standard_normal((n, hd))
    # scale the scores to the requested spread while keeping |s| <= M
    scale = spread / np.sqrt(hd)
    M = scale * hd  # = scale * |q| |k|, the Cauchy-Schwarz bound
    o, smax = oracle.attend(q, K, V, scale)
    s = scale * K @ q
    assert np.all(np.abs(s) <= M * (1 + 1e-12))
    p = np.exp(s - M)  # fixed shift, no running max
    fixed = (p[:, None] * V).sum(0) / p.sum()
    # chunks reduced independently with the same shift give the same result
    parts = [(np.exp(s[a:a + 37] - M)[:, None] * V[a:a + 37]).sum(0) for a in range(0, n, 37)]
    ls = [np.exp(s[a:a + 37] - M).sum() for a in range(0, n, 37)]
    chunked = sum(parts) / sum(ls)
    lib = scipy.special.softmax(s) @ V
    assert np.allclose(o, fixed, rtol=1e-12, atol=1e-14)
    assert np.allclose(o, chunked, rtol=1e-12, atol=1e-14)
    assert np.allclose(o, lib, rtol=1e-12, atol=1e-14)
    assert smax == pytest.approx(s.max(), abs=1e-12)


def test_attend_adversarial_scores():
    # scores at both ends of the bound: exp(s - M) spans e^-2M .. 1
    hd = 16
    q = np.zeros(hd); q[0] = 4.0
    K = np.zeros((3, hd)); K[0, 0] = 4.0; K[1, 0] = -4.0; K[2, 0] = 0.0
    V = np.eye(3, hd)
    o, _ = oracle.attend(q, K, V, 1.0)
    s = np.array([16.0, -16.0, 0.0])
    assert np.allclose(o, scipy.special.softmax(s) @ V, rtol=1e-14, atol=1e-300)


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(5)
    for trial in range(300):
        n, k = 256, 8
        logits = rng.standard_normal(n)
        if trial % 3 == 0:  # exact ties, also across the k-th boundary
            logits = np.round(logits * 2) / 2
        ids, w, gap = oracle.topk(logits, k)
        order = np.lexsort((np.arange(n), -logits))  # value desc, then index asc
        assert list(ids) == list(order[:k])
        assert gap == pytest.approx(logits[order[k - 1]] - logits[order[k]], abs=0)
        assert np.allclose(w, scipy.special.softmax(logits[order[:k]]), rtol=1e-14)
        assert w.sum() == pytest.approx(1.0, abs=1e-14)


def test_rmsnorm_and_silu_vs_torch():
    rng = np.random.default_rng(6)
    for n in (16, 64, 512):
        x = rng.standard_normal(n) * 3
        g = rng.uniform(0.8, 1.2, n).astype(np.float32)
        assert np.allclose(oracle.rmsnorm(x, g, 1e-6), rmsnorm_ref(x, g, 1e-6), rtol=1e-13)
        c = np.full(n, -2.5)  # constant row: g * sign(c)
        assert np.allclose(oracle.rmsnorm(c, g, 1e-12), -g.astype(np.float64), rtol=1e-12)
    a = np.linspace(-20, 20, 401)
    got = np.array([oracle.lib().msk_or_silu(float(v)) for v in a])
    assert np.allclose(got, torch.nn.functional.silu(torch.from_numpy(a)).numpy(), rtol=1e-14, atol=1e-300)


# ---- hand-computable one-layer / four-expert cases ----------------------------
def _hand(P=7, gq=1.0, gk=1.0, **over):
    w = hand_workload(past=P)
    d = 16
    z = np.zeros((d, d))
    eye = np.eye(d)
    rng = np.random.default_rng(7)
    weights = {
        "attn_norm_g": np.ones(d, np.float32), "moe_norm_g": np.ones(d, np.float32),
        "q_norm_g": np.full(d, gq, np.float32), "k_norm_g": np.full(d, gk, np.float32),
        "router": np.zeros((4, d), np.float32),
        "wq": z, "wk": z, "wv": eye, "wo": z,
        "w_gate": [z] * 4, "w_up": [z] * 4, "w_down": [z] * 4,
    }
    weights.update(over)
    past_k = e4m3_codes(rng.standard_normal((P, d)))
    past_v = e4m3_codes(rng.standard_normal((P, d)))
    pk = over.pop("_past_k", None)
    return w, weights, past_k, past_v, rng


def _run(w, weights, past_k, past_v, h_in, forced=None):
    m = HandModel(w, weights, [[[past_k]]], [[[past_v]]])
    return oracle.step(w, m.src.ptr, h_in, w.positions(), forced_ids=forced, threads=1)


def test_hand_zero_query_attends_uniformly():
    # W_q = 0 -> q = 0 after QK-norm -> all scores 0 -> output = mean of V
    w, weights, pk, pv, rng = _hand()
    h = bf16_bits(rng.standard_normal((1, 16)) + 0.5)
    o = _run(w, weights, pk, pv, h)
    x = rmsnorm_ref(bf16_values(h), weights["attn_norm_g"], w.rms_eps)
    v_new = e4m3_codes(x @ weights["wv"].T)  # W_v = I
    V = np.vstack([e4m3_values(pv), e4m3_values(v_new)])
    assert np.array_equal(o["v_new"][0, 0], v_new[0])
    assert np.allclose(o["attn_out"][0, 0], V.mean(0), rtol=1e-13, atol=1e-15)
    # W_o = 0 and zero experts: the residual passes through unchanged
    assert np.array_equal(o["hidden_out"], h)


def test_hand_dominant_key():
    # q along e0 with gain 3, one past key 8*e0: its score is 24, all others 0
    P = 9
    w, weights, pk, pv, rng = _hand(P=P, gq=3.0)
    wq = np.zeros((16, 16)); wq[0, :] = 1.0
    weights["wq"] = wq
    kv = e4m3_values(pk).copy()
    kv[:, 0] = 0.0
    kv[4, 0] = 8.0
    pk = e4m3_codes(kv)
    h = bf16_bits(np.abs(rng.standard_normal((1, 16))) + 0.1)  # sum(x) > 0
    o = _run(w, weights, pk, pv, h)
    assert np.allclose(o["attn_out"][0, 0], e4m3_values(pv)[4], rtol=0, atol=1e-8)
    x = rmsnorm_ref(bf16_values(h), weights["attn_norm_g"], w.rms_eps)[0]
    q0 = x.sum()
    s_star = 3.0 * q0 / np.sqrt(q0 * q0 / 16 + w.rms_eps) * 8.0 / 4.0  # ~24
    assert o["s_max_minus_bound"][0] == pytest.approx(s_star - 4 * 3.0 * 1.0, rel=1e-13)


def test_hand_residual_with_zero_experts():
    # experts all zero: h_out = h_in + attn . W_o^T exactly
    w, weights, pk, pv, rng = _hand()
    wo = np.zeros((16, 16)); wo[np.arange(16), (np.arange(16) * 5) % 16] = 0.5
    weights["wo"] = wo
    weights["wq"] = np.eye(16)
    weights["wk"] = np.eye(16) * -1.0
    h = bf16_bits(rng.standard_normal((1, 16)))
    o = _run(w, weights, pk, pv, h)
    want = bf16_values(h) + o["attn_out"][0] @ wo.T
    assert np.allclose(o["h_out"], want, rtol=1e-14, atol=1e-14)


def test_hand_single_expert_swiglu_closed_form():
    # router logit_e = c_e * x2[0] with c = (3, 1, 2, 0) and x2[0] > 0 -> experts
    # (0, 2); expert 2 is all zero; expert 0: gate = x2, up = 2 x2, down = I.
    w, weights, pk, pv, rng = _hand()
    eye, z = np.eye(16), np.zeros((16, 16))
    router = np.zeros((4, 16), np.float32)
    router[:, 0] = [3, 1, 2, 0]
    weights.update(router=router, w_gate=[eye, z, z, z], w_up=[2 * eye, z, z, z], w_down=[eye, z, z, z])
    hv = rng.standard_normal((1, 16))
    hv[0, 0] = abs(hv[0, 0]) + 0.5
    h = bf16_bits(hv)
    o = _run(w, weights, pk, pv, h)
    x2 = rmsnorm_ref(bf16_values(h), weights["moe_norm_g"], w.rms_eps)[0]
    assert list(o["route_ids"][0, 0]) == [0, 2]
    w0 = 1.0 / (1.0 + np.exp(-x2[0]))  # softmax of (3 x0, 2 x0) at expert 0
    assert o["route_w"][0, 0, 0] == pytest.approx(w0, rel=1e-14)
    y = torch.nn.functional.silu(torch.from_numpy(x2)).numpy() * 2 * x2
    assert np.allclose(o["h_out"][0], bf16_values(h)[0] + w0 * y, rtol=1e-13, atol=1e-14)


def test_hand_router_ties_break_by_index():
    w, weights, pk, pv, rng = _hand()
    router = np.zeros((4, 16), np.float32)
    router[:, 0] = [1, 1, 0.5, 1]
    weights["router"] = router
    hv = np.abs(rng.standard_normal((1, 16))) + 0.1
    o = _run(w, weights, pk, pv, bf16_bits(hv))
    assert list(o["route_ids"][0, 0]) == [0, 1]
    assert o["route_gap"][0, 0] == 0.0
    assert np.allclose(o["route_w"][0, 0], [0.5, 0.5], rtol=1e-15)


def test_forced_routing_overrides():
    w, weights, pk, pv, rng = _hand()
    router = np.zeros((4, 16), np.float32)
    router[:, 0] = [3, 1, 2, 0]
    weights["router"] = router
    hv = np.abs(rng.standard_normal((1, 16))) + 0.1
    forced = np.array([[[3, 1]]], np.int16)
    o = _run(w, weights, pk, pv, bf16_bits(hv), forced=forced)
    assert list(o["route_ids"][0, 0]) == [3, 1]
    lg = o["logits"][0, 0]
    assert np.allclose(o["route_w"][0, 0], scipy.special.softmax(lg[[3, 1]]), rtol=1e-14)


# ---- step invariants on a small generated model --------------------------------
@pytest.fixture(scope="module")
def mini():
    w = mini_workload()
    return w, ExtendableSource(w)


def test_verify_equals_sequential_decode(mini):
    w, src0 = mini
    hid = synth.host_hidden(w)
    ver = oracle.step(w, src0.src.ptr, hid, w.positions(), threads=2)
    seq = ExtendableSource(w, src0.arrays)
    tps = w.tokens_per_seq
    for i in range(tps):
        rows = [b * tps + i for b in range(w.n_seqs)]
        pos = np.array([[w.past + i] for _ in range(w.n_seqs)], np.int32)
        o = oracle.step(w.with_(tokens_per_seq=1), seq.src.ptr, hid[rows], pos, threads=2)
        assert np.array_equal(o["h_out"], ver["h_out"][rows])
        assert np.array_equal(o["attn_out"], ver["attn_out"][:, rows])
        assert np.array_equal(o["route_ids"], ver["route_ids"][:, rows])
        for l in range(w.n_layers):
            kvd = w.n_kv_heads * w.head_dim
            for b in range(w.n_seqs):
                kn = o["k_new"][l, b].reshape(w.n_kv_heads, w.head_dim)
                vn = o["v_new"][l, b].reshape(w.n_kv_heads, w.head_dim)
                assert np.array_equal(o["k_new"][l, b], ver["k_new"][l, rows[b]]) and kvd
                for h in range(w.n_kv_heads):
                    seq.append(l, b, h, kn[h], vn[h])
        seq.rebuild()


def test_window_longer_than_context_equals_full(mini):
    w, src = mini
    hid = synth.host_hidden(w)
    wide = w.with_(window=w.past + w.tokens_per_seq)  # every key inside the window
    a = oracle.step(wide, src.src.ptr, hid, w.positions(), threads=2)
    b = oracle.step(wide.with_(sliding=[0, 0]), src.src.ptr, hid, w.positions(), threads=2)
    assert np.array_equal(a["h_out"], b["h_out"])
    # and a short window does change the sliding layer
    c = oracle.step(w, src.src.ptr, hid, w.positions(), threads=2)
    assert not np.array_equal(c["attn_out"][0], a["attn_out"][0])
    assert np.array_equal(c["attn_out"][0][:, :0], a["attn_out"][0][:, :0])


def test_window_masks_exactly_the_old_keys(mini):
    # with window W the sliding layer's output must not depend on keys older
    # than pos - W + 1: scrambling them changes nothing
    w, src = mini
    hid = synth.host_hidden(w)
    a = oracle.step(w, src.src.ptr, hid, w.positions(), threads=2)
    alt = ExtendableSource(w, src.arrays)
    lo = w.past - w.window + 1  # oldest key the first block token may see
    for (l, b, h), (k, v) in list(alt.past.items()):
        if l == 0:
            k, v = k.copy(), v.copy()
            k[:lo] = 0x38
            v[:lo] = 0x40
            alt.past[(l, b, h)] = (k, v)
    alt.rebuild()
    b_ = oracle.step(w, alt.src.ptr, hid, w.positions(), threads=2)
    assert np.array_equal(a["attn_out"][0], b_["attn_out"][0])


def test_sequences_are_independent(mini):
    w, src = mini
    hid = synth.host_hidden(w)
    both = oracle.step(w, src.src.ptr, hid, w.positions(), threads=2)
    tps = w.tokens_per_seq
    for b in range(w.n_seqs):
        rows = list(range(b * tps, (b + 1) * tps))
        one = oracle.step(w.with_(n_seqs=1), src.src.ptr, hid[rows], [w.positions()[b]], seq_ids=[b],
                          threads=1)
        assert np.array_equal(one["h_out"], both["h_out"][rows])


def test_lazy_source_equals_arrays(mini):
    w, src = mini
    hid = synth.host_hidden(w)
    lazy = synth.LazySource(w)
    a = oracle.step(w, lazy.ptr, hid, w.positions(), threads=2)
    b = oracle.step(w, src.src.ptr, hid, w.positions(), threads=2)
    assert np.array_equal(a["h_out"], b["h_out"])
    assert np.array_equal(a["hidden_out"], b["hidden_out"])


def test_forced_kv_code_is_used():
    # uniform attention (W_q = 0): forcing the new token's v codes changes the
    # mean by exactly the forced values' share
    w, weights, pk, pv, rng = _hand()
    h = bf16_bits(rng.standard_normal((1, 16)) + 0.5)
    m = HandModel(w, weights, [[[pk]]], [[[pv]]])
    a = oracle.step(w, m.src.ptr, h, w.positions(), threads=1)
    fv = np.full((1, 1, 16), -1, np.int16)
    fv[0, 0, 3] = 0x40  # 2.0
    b = oracle.step(w, m.src.ptr, h, w.positions(), forced_v=fv, threads=1)
    n = w.past + 1
    delta = (2.0 - e4m3_values(a["v_new"][0, 0, 3:4])[0]) / n
    assert b["attn_out"][0, 0, 3] == pytest.approx(a["attn_out"][0, 0, 3] + delta, rel=1e-13)
    assert np.array_equal(np.delete(b["attn_out"][0, 0], 3), np.delete(a["attn_out"][0, 0], 3))
    assert b["v_new"][0, 0, 3] == 0x40
    assert np.allclose(a["v_pre"][0, 0], rmsnorm_ref(bf16_values(h), weights["attn_norm_g"], w.rms_eps)[0])
