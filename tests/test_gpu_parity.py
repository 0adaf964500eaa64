"""GPU parity: the CUDA step (through the C ABI) against the fp64 oracle.

Tolerances are the target's: routing sets identical unless the oracle's
8th-9th logit gap is below 1e-3 (then the oracle is replayed with the GPU's
routing for that token), final hidden states max-abs <= 2e-2 and rel-L2 <=
1e-2, per-layer attention outputs rel-L2 <= 5e-3.  Sizes: the tiny, 8-layer
decode and 8-layer verify workloads in full; a ragged multi-sequence case
(different past lengths, an empty past, a window shorter than the context,
chunk boundaries crossed); the long-context and largest workloads at full
size in the benchmark's launch configuration, with the oracle on sampled
sequences.
"""
import numpy as np
import pytest
import torch

import synth
import synth.gpu as sg
import verify_step_megakernel_b200 as msk
from synth.configs import Workload
from synth.engine import Engine
from tests._parity import assert_parity, bf16_to_f64, run_parity

pytestmark = pytest.mark.gpu


def _report(name, rep):
    k, v = rep["kv_k"], rep["kv_v"]
    print(f"\n[{name}] attn_rel max {max(rep['attn_rel']):.2e}  h_abs {rep['h_abs']:.2e}  h_rel {rep['h_rel']:.2e}"
          f"  dh_rel {rep['dh_rel']:.2e}  route exempt {rep['n_exempt']} forced {rep['forced']}"
          f"  route_w abs {rep['route_w_abs']:.2e} rel {rep['route_w_rel']:.2e}"
          f"  kv straddles {rep['forced_kv']}/{rep['kv_codes']} (expected {k['expected_diff'] + v['expected_diff']:.0f})"
          f"  encoder mismatches {k['enc_mismatch'] + v['enc_mismatch']}"
          f"  pre rel-L2 max K {max(k['pre_rel']):.2e} V {max(v['pre_rel']):.2e}  invalid {rep['kv_invalid']}")


def _kv_written_match(w, eng, ref, positions, seqs):
    """The fp8 K/V this step wrote equal the oracle's codes up to one e4m3
    step where the fp32 and fp64 values straddle a rounding boundary."""
    tps = len(positions[0])
    kvd = w.n_kv_heads * w.head_dim
    tot = same = 0
    for l in range(w.n_layers):
        for i, b in enumerate(seqs):
            k, v = eng.read_kv(l, b, positions[b][0], tps)
            for arr, key in ((k, "k_new"), (v, "v_new")):
                want = ref[key][l, i * tps:(i + 1) * tps].reshape(tps, kvd)
                tot += want.size
                same += int((arr == want).sum())
                a = torch.from_numpy(arr).view(torch.float8_e4m3fn).double().numpy()
                bb = torch.from_numpy(want).view(torch.float8_e4m3fn).double().numpy()
                assert np.all(np.abs(a - bb) <= np.maximum(np.abs(bb), 2.0 ** -6) * 0.125 + 1e-12)
    assert same / tot > 0.9, same / tot


@pytest.mark.parametrize("name", ["tiny", "dec8", "ver8"])
def test_parity_tensor_core_experts(name):
    """The same parity bar with gate/up on the block-scaled tensor cores
    (MSK_F_TC_EXPERTS): NVFP4 weights as stored, activations as e2m1 terms."""
    w = synth.WORKLOADS[name]
    eng = Engine(w, flags=msk.F_TC_EXPERTS)
    eng.fill_past()
    hid = sg.hidden(w)
    rep, gpu, ref = run_parity(w, eng, hid, w.positions())
    _report(name + " tc", rep)
    assert_parity(rep)
    eng.close()


@pytest.mark.parametrize("name", ["tiny", "dec8", "ver8"])
def test_parity_cuda_core_experts(name):
    """Every expert unit's gate/up on the CUDA-core path (tau above the unit size)."""
    w = synth.WORKLOADS[name]
    eng = Engine(w, tau=msk.TAU_NEVER)
    eng.fill_past()
    hid = sg.hidden(w)
    rep, gpu, ref = run_parity(w, eng, hid, w.positions())
    _report(name + " cc", rep)
    assert_parity(rep)
    eng.close()


@pytest.mark.parametrize("name", ["tiny", "dec8", "ver8"])
def test_parity_workload(name):
    w = synth.WORKLOADS[name]
    eng = Engine(w)
    eng.fill_past()
    hid = sg.hidden(w)
    pos = w.positions()
    rep, gpu, ref = run_parity(w, eng, hid, pos)
    _report(name, rep)
    assert_parity(rep)
    _kv_written_match(w, eng, ref, pos, list(range(w.n_seqs)))
    eng.close()


@pytest.mark.parametrize("tau", [2, 3])
def test_parity_mixed_expert_paths(tau):
    """expert_mma_min_tokens = tau: in one step, the gate/up of expert units
    with at least tau tokens runs on the block-scaled tensor cores and the
    rest on the CUDA-core path; both kinds occur in every layer here."""
    w = synth.WORKLOADS["ver8"]
    eng = Engine(w, tau=tau)
    eng.fill_past()
    hid = sg.hidden(w)
    rep, gpu, ref = run_parity(w, eng, hid, w.positions())
    _report(f"ver8 tau {tau}", rep)
    assert_parity(rep)
    # both paths ran: per layer, experts chosen by at least tau tokens and by fewer
    for l in range(w.n_layers):
        cnt = np.bincount(gpu["route_ids"][l].ravel().astype(np.int64), minlength=w.n_experts)
        assert (cnt >= tau).any() and ((cnt > 0) & (cnt < tau)).any(), (l, np.bincount(cnt))
    assert msk.msk_query(eng.h).repacked_bytes > 0
    eng.close()


RAGGED = Workload("ragged", 3, 256, 4, 2, 64, 128, [1, 0, 1], 3, 3, 0, 0x5EED + 40, n_experts=32, top_k=4,
                  window=100)


@pytest.mark.parametrize("tau", [msk.TAU_NEVER, 1], ids=["cuda_core", "tensor_core"])
def test_parity_ragged_sequences(tau):
    w = RAGGED
    past = [0, 130, 517]  # empty past, a chunk boundary crossed, window < context
    eng = Engine(w, past_per_seq=past, tau=tau)
    eng.fill_past()
    hid = sg.hidden(w)
    pos = [[p + i for i in range(w.tokens_per_seq)] for p in past]
    rep, gpu, ref = run_parity(w, eng, hid, pos)
    _report("ragged", rep)
    assert_parity(rep)
    _kv_written_match(w, eng, ref, pos, [0, 1, 2])
    eng.close()


def test_hd128_window_edge_and_single_token_window():
    # window 1: each query sees only itself; 128-wide heads, GQA group 4
    w = Workload("w1", 2, 512, 8, 2, 128, 256, [1, 1], 2, 2, 300, 0x5EED + 41, n_experts=64, top_k=8, window=1)
    eng = Engine(w)
    eng.fill_past()
    hid = sg.hidden(w)
    rep, gpu, ref = run_parity(w, eng, hid, w.positions())
    _report("w1", rep)
    assert_parity(rep)
    eng.close()


def test_step_is_deterministic_and_repeatable():
    w = synth.WORKLOADS["ver8"].with_(n_layers=2, sliding=[1, 0])
    eng = Engine(w)
    eng.fill_past()
    hid = sg.hidden(w)
    a = eng.step(hid, w.positions())
    b = eng.step(hid, w.positions())
    assert a["status"] == 0 and b["status"] == 0
    assert np.array_equal(a["hidden_out"], b["hidden_out"])
    assert np.array_equal(a["attn_out"], b["attn_out"])
    eng.close()


def test_bad_positions_are_reported():
    w = synth.WORKLOADS["tiny"].with_(n_seqs=1, tokens_per_seq=2)
    eng = Engine(w)
    hid = sg.hidden(w)
    r = eng.step(hid, [[5, 7]])  # not contiguous
    assert r["status"] == msk.MskError(6, "").code
    r = eng.step(hid, [[w.past + 100, w.past + 101]])  # beyond the (rounded-up) capacity
    assert r["status"] == 6
    r = eng.step(hid, [[3, 4]])
    assert r["status"] == 0
    eng.close()


def test_invalid_arguments_and_bound():
    w = synth.WORKLOADS["tiny"]
    wts = sg.DeviceWeights(w)
    from synth.engine import config_struct, layer_structs
    cfg = config_struct(w)
    cfg.head_dim = 96
    with pytest.raises(msk.MskError) as e:
        msk.msk_create(cfg, layer_structs(wts), 0)
    assert e.value.code == 2
    cfg = config_struct(w)
    layers = layer_structs(wts)
    big = torch.full((w.head_dim,), 2.0, dtype=torch.float32, device="cuda")  # M = 8*2*2 = 32: 2M = 64 ok
    layers[0].q_norm_g = big.data_ptr()
    h = msk.msk_create(cfg, layers, 0)
    msk.msk_destroy(h)
    bigger = torch.full((w.head_dim,), 2.5, dtype=torch.float32, device="cuda")  # M = 50: 2M >= 80
    layers[0].q_norm_g = bigger.data_ptr()
    layers[0].k_norm_g = bigger.data_ptr()
    with pytest.raises(msk.MskError) as e:
        msk.msk_create(cfg, layers, 0)
    assert e.value.code == 5
    layers = layer_structs(wts)
    layers[1].wq.codes = layers[1].wq.codes + 1  # misaligned
    with pytest.raises(msk.MskError) as e:
        msk.msk_create(cfg, layers, 0)
    assert e.value.code == 1


@pytest.mark.slow
def test_parity_long_context_sampled():
    w = synth.WORKLOADS["long"]
    eng = Engine(w)
    eng.fill_past()
    hid = sg.hidden(w)
    rep, gpu, ref = run_parity(w, eng, hid, w.positions())
    _report("long", rep)
    assert_parity(rep)
    eng.close()


@pytest.mark.slow
def test_parity_largest_sampled():
    w = synth.WORKLOADS["large"]
    eng = Engine(w)
    eng.fill_past()
    hid = sg.hidden(w)
    rep, gpu, ref = run_parity(w, eng, hid, w.positions(), seqs=[0, 15])
    _report("large", rep)
    assert_parity(rep)
    eng.close()


def test_routing_exact_ties_break_by_lower_index():
    # router rows equal in groups of three (row r = row 3 (r // 3)), so every
    # token's logits come in exactly equal triples and the cut after the 8th
    # pick falls inside a triple: only the tie rule (lower expert index
    # first) decides which two of its three experts are taken.  The device
    # router is overwritten in place (the handle borrows it); the oracle reads
    # the same values from an array source.
    from tests._models import ExtendableSource

    w = synth.WORKLOADS["tiny"].with_(n_seqs=1, tokens_per_seq=1)
    eng = Engine(w)
    eng.fill_past()
    src = ExtendableSource(w)
    E, d = w.n_experts, w.d_model
    for l in range(w.n_layers):
        r = src.arrays["vec"][(l, "router")].reshape(E, d)
        tied = np.ascontiguousarray(r[(np.arange(E) // 3) * 3].reshape(-1)).astype(np.float32)
        src.arrays["vec"][(l, "router")] = tied
        ptr = eng.wts.layers[l]["router"]
        dev_t = next(t for t in eng.wts.keep if t.data_ptr() == ptr)
        dev_t.copy_(torch.from_numpy(tied))
    src.rebuild()
    hid = sg.hidden(w)
    rep, gpu, ref = run_parity(w, eng, hid, w.positions(), src=src.src)
    _report("ties", rep)
    # the oracle's 8th-9th gap is exactly 0 here, so compare the picks
    # themselves instead of exempting them
    for l in range(w.n_layers):
        assert ref["route_gap"][l, 0] == 0.0  # the 8th and 9th logits are equal
        got = sorted(int(x) for x in gpu["route_ids"][l, 0])
        assert got == sorted(int(x) for x in ref["route_ids"][l, 0]), (l, got, ref["route_ids"][l, 0])
        # among the experts tied with the 8th logit, the lowest indices won
        lg = gpu["logits"][l, 0]
        v8 = min(lg[e] for e in got)
        tied = sorted(int(e) for e in np.nonzero(lg == v8)[0])
        taken = [e for e in got if lg[e] == v8]
        assert len(tied) > len(taken) and taken == tied[:len(taken)], (l, tied, taken)
    assert rep["forced"] == 0
    assert rep["h_abs"] <= 2e-2 and rep["h_rel"] <= 1e-2, rep
    assert max(rep["attn_rel"]) <= 5e-3
    eng.close()


def _set_router(eng, w, fn):
    """Overwrite every layer's device router [E][d] with fn(original)."""
    E, d = w.n_experts, w.d_model
    for l in range(w.n_layers):
        ptr = eng.wts.layers[l]["router"]
        dev_t = next(t for t in eng.wts.keep if t.data_ptr() == ptr)
        r = dev_t.view(E, d).cpu().numpy()
        dev_t.copy_(torch.from_numpy(np.ascontiguousarray(fn(r), dtype=np.float32).reshape(-1)))


def test_routing_all_logits_equal_picks_the_first_k():
    # one router row for every expert: all logits of a token are equal, so
    # the picks are experts 0 .. k-1 with weights exactly 1/k
    w = synth.WORKLOADS["tiny"].with_(n_seqs=2, tokens_per_seq=2)
    eng = Engine(w)
    eng.fill_past()
    _set_router(eng, w, lambda r: np.repeat(r[:1], r.shape[0], axis=0))
    out = eng.step(sg.hidden(w), w.positions())
    assert out["status"] == 0
    k = w.top_k
    for l in range(w.n_layers):
        for t in range(w.T):
            assert sorted(int(x) for x in out["route_ids"][l, t]) == list(range(k))
            assert np.all(out["route_w"][l, t] == np.float32(1.0 / k))
    assert np.isfinite(bf16_to_f64(out["hidden_out"])).all()
    eng.close()


def test_routing_nan_logit_is_never_picked():
    # a NaN router row makes that expert's logit NaN for every token; it
    # ranks last, so it is never among the picks and nothing NaN reaches
    # the hidden state
    w = synth.WORKLOADS["tiny"].with_(n_seqs=2, tokens_per_seq=2)
    eng = Engine(w)
    eng.fill_past()
    bad = 5

    def poison(r):
        r = r.copy()
        r[bad] = np.nan
        return r

    _set_router(eng, w, poison)
    out = eng.step(sg.hidden(w), w.positions())
    assert out["status"] == 0
    assert np.isnan(out["logits"][:, :, bad]).all()
    assert not (out["route_ids"] == bad).any()
    assert np.isfinite(out["route_w"]).all()
    assert np.isfinite(bf16_to_f64(out["hidden_out"])).all()
    eng.close()
