"""Comparisons of a GPU step with the oracle, with the tolerances of the
target: routing sets exact unless the oracle's 8th-9th logit gap is below
1e-3; final hidden max-abs 2e-2 and rel-L2 1e-2; attention output rel-L2
5e-3 per layer."""
import numpy as np

import oracle
import synth
import verify_step_megakernel_b200 as msk

TOL_ATTN_REL = 5e-3
TOL_H_ABS = 2e-2
TOL_H_REL = 1e-2
GAP_EXEMPT = 1e-3


def bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def compare(w, gpu, ref, h_in_bits, rows=None):
    """Compare one GPU step with the oracle; returns a report dict (no asserts).
    rows: GPU token rows the oracle covered (default all)."""
    rows = list(range(gpu["hidden_out"].shape[0])) if rows is None else rows
    L, k = w.n_layers, w.top_k
    rep = {"route_mismatch": [], "attn_rel": [], "n_exempt": 0}
    for l in range(L):
        for i, t in enumerate(rows):
            a = set(int(x) for x in gpu["route_ids"][l, t])
            b = set(int(x) for x in ref["route_ids"][l, i])
            if a != b:
                if ref["route_gap"][l, i] < GAP_EXEMPT:
                    rep["n_exempt"] += 1
                else:
                    rep["route_mismatch"].append((l, t, sorted(a), sorted(b), float(ref["route_gap"][l, i])))
        rep["attn_rel"].append(rel_l2(gpu["attn_out"][l][rows], ref["attn_out"][l]))
    # routing weights, matched by expert id where the sets agree
    gw, rw = [], []
    for l in range(L):
        for i, t in enumerate(rows):
            a = {int(e): float(x) for e, x in zip(gpu["route_ids"][l, t], gpu["route_w"][l, t])}
            b = {int(e): float(x) for e, x in zip(ref["route_ids"][l, i], ref["route_w"][l, i])}
            if set(a) == set(b):
                gw += [a[e] for e in sorted(a)]
                rw += [b[e] for e in sorted(b)]
    rep["route_w_abs"] = float(np.abs(np.subtract(gw, rw)).max()) if gw else 0.0
    rep["route_w_rel"] = rel_l2(gw, rw) if gw else 0.0
    h_gpu = bf16_to_f64(gpu["hidden_out"][rows])
    h_ref = ref["h_out"]
    h_in = bf16_to_f64(h_in_bits)
    rep["h_abs"] = float(np.abs(h_gpu - h_ref).max())
    rep["h_rel"] = rel_l2(h_gpu, h_ref)
    rep["dh_rel"] = rel_l2(h_gpu - h_in, h_ref - h_in)
    return rep


def forced_from_gpu(w, gpu, ref, rows):
    """Oracle forced-routing input: the GPU's ids where routing differs only
    at exempt near-ties (oracle gap < 1e-3), else -1 (oracle's own)."""
    L, k = w.n_layers, w.top_k
    fr = np.full((L, len(rows), k), -1, np.int16)
    for l in range(L):
        for i, t in enumerate(rows):
            if set(gpu["route_ids"][l, t]) != set(ref["route_ids"][l, i]) and ref["route_gap"][l, i] < GAP_EXEMPT:
                fr[l, i] = gpu["route_ids"][l, t]
    return fr


# fp8 KV codes.  The GPU encodes its own fp32 K/V value g, the oracle its
# fp64 value x of the same quantity; both round to nearest even on the e4m3
# grid.  Where a rounding boundary lies between g and x the two codes differ,
# and both are correct roundings of a correct value (g is within the step's
# error of x).  The checks, in order:
#  1. every code the GPU wrote equals the oracle's encoder applied to the
#     GPU's own captured fp32 value -- bit-exact, integer work;
#  2. the GPU's pre-encoding values match the oracle's to rel-L2
#     KV_PRE_REL per layer.  K and V are linear in the layer's normed input,
#     so their relative error is that of the hidden state entering the
#     layer, which the target bounds by its hidden-state tolerance (1e-2);
#  3. the codes that differ are then exactly those where enc(g) != enc(x);
#     their number must stay within KV_STRADDLE_SLACK times the expected
#     count of boundary crossings, sum_i |g_i - x_i| / step(x_i) (a boundary
#     falls between g and x with probability |g - x| / step), plus a few.
# Differing codes pass checks 1-3 only as valid roundings; the oracle is then
# replayed with the GPU's codes at those places, like near-tied routing.
KV_PRE_REL = 1e-2
KV_STRADDLE_SLACK = 3.0
# Routing weights scale the expert outputs added to the hidden state: they
# are held to the hidden state's tolerances.
ROUTE_W_ABS = 2e-2
ROUTE_W_REL = 1e-2


def _e4m3(codes):
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def e4m3_step(x):
    """Spacing of the e4m3 grid at |x| (2^-9 below the normal range)."""
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.exp2(e - 3)


def kv_check(ref_pre, gpu_codes, gpu_pre):
    """(forced codes or -1, report): checks 1-3 above for one of K or V,
    arrays [L][T][Hkv*hd]; the oracle's own codes are its encoder applied to
    its pre-values."""
    enc = oracle.e4m3_encode(np.asarray(gpu_pre, np.float64))
    ref_codes = oracle.e4m3_encode(ref_pre)
    rep = {"enc_mismatch": int((enc != gpu_codes).sum())}
    L = ref_pre.shape[0]
    rep["pre_rel"] = [rel_l2(gpu_pre[l], ref_pre[l]) for l in range(L)]
    diff = ref_codes != gpu_codes
    rep["n_diff"] = int(diff.sum())
    rep["expected_diff"] = float(np.minimum(1.0, np.abs(gpu_pre - ref_pre) / e4m3_step(ref_pre)).sum())
    forced = np.full(ref_codes.shape, -1, np.int16)
    forced[diff] = gpu_codes[diff]
    return forced, rep


def kv_report_ok(rep):
    return (rep["enc_mismatch"] == 0 and max(rep["pre_rel"]) <= KV_PRE_REL
            and rep["n_diff"] <= KV_STRADDLE_SLACK * rep["expected_diff"] + 8)


def gpu_kv_codes(eng, w, positions, seqs):
    """K/V codes the GPU step wrote at the step's positions: [L][T][Hkv*hd]."""
    tps = len(positions[0])
    kvd = w.n_kv_heads * w.head_dim
    K = np.zeros((w.n_layers, len(seqs) * tps, kvd), np.uint8)
    V = np.zeros_like(K)
    for l in range(w.n_layers):
        for i, b in enumerate(seqs):
            k, v = eng.read_kv(l, b, positions[b][0], tps)
            K[l, i * tps:(i + 1) * tps] = k
            V[l, i * tps:(i + 1) * tps] = v
    return K, V


def run_parity(w, eng, gpu_hidden, positions, seqs=None, threads=None, max_replays=4, src=None):
    """Oracle on sequences `seqs` (default all) of the step; returns (report,
    gpu outputs, oracle outputs).  Decisions with two valid answers (routing
    near-ties, fp8 codes whose GPU and oracle values straddle a rounding
    boundary, see above) are replayed in the oracle with the GPU's choice so
    the layers after them stay comparable; every other difference counts
    against the tolerances.  src: the oracle's input source (default the
    workload's generator; an array source where a test changed the device
    weights)."""
    seqs = list(range(len(positions))) if seqs is None else seqs
    tps = len(positions[0])
    h_bits = gpu_hidden.cpu().numpy().view(np.uint16)
    gpu = eng.step(gpu_hidden, positions)
    assert gpu["status"] == 0, msk.STATUS.get(gpu["status"])
    rows = [b * tps + i for b in seqs for i in range(tps)]
    gk, gv = gpu_kv_codes(eng, w, positions, seqs)
    gk_pre = gpu["k_pre"][:, rows].astype(np.float64)
    gv_pre = gpu["v_pre"][:, rows].astype(np.float64)
    src = synth.LazySource(w) if src is None else src
    pos_s = [positions[b] for b in seqs]
    ww = w.with_(n_seqs=len(seqs))
    kw = dict(seq_ids=seqs, threads=threads)
    ref = oracle.step(ww, src.ptr, h_bits[rows], pos_s, **kw)
    fr = fk = fv = None
    for _ in range(max_replays):
        nfr = forced_from_gpu(ww, gpu, ref, rows)
        nfk, _ = kv_check(ref["k_pre"], gk, gk_pre)
        nfv, _ = kv_check(ref["v_pre"], gv, gv_pre)
        if fr is not None:  # keep earlier decisions
            nfr = np.where(nfr >= 0, nfr, fr)
            nfk = np.where(nfk >= 0, nfk, fk)
            nfv = np.where(nfv >= 0, nfv, fv)
        if fr is not None and np.array_equal(nfr, fr) and np.array_equal(nfk, fk) and np.array_equal(nfv, fv):
            break
        if not ((nfr >= 0).any() or (nfk >= 0).any() or (nfv >= 0).any()):
            break
        fr, fk, fv = nfr, nfk, nfv
        ref = oracle.step(ww, src.ptr, h_bits[rows], pos_s, forced_ids=fr, forced_k=fk, forced_v=fv, **kw)
    # the KV checks against the oracle's final (replayed) pre-values: a
    # forced code never changes the pre-values of its own layer
    _, krep = kv_check(ref["k_pre"], gk, gk_pre)
    _, vrep = kv_check(ref["v_pre"], gv, gv_pre)
    rep = compare(ww, gpu, ref, h_bits[rows], rows)
    rep["forced"] = 0 if fr is None else int((fr[..., 0] >= 0).sum())
    rep["forced_kv"] = 0 if fk is None else int((fk >= 0).sum() + (fv >= 0).sum())
    rep["kv_codes"] = int(gk.size + gv.size)
    rep["kv_k"], rep["kv_v"] = krep, vrep
    rep["kv_invalid"] = int(not kv_report_ok(krep)) + int(not kv_report_ok(vrep))
    return rep, gpu, ref


def assert_parity(rep):
    assert not rep["route_mismatch"], rep["route_mismatch"][:5]
    assert rep.get("kv_invalid", 0) == 0, (rep.get("kv_k"), rep.get("kv_v"))
    assert rep["route_w_abs"] <= ROUTE_W_ABS and rep["route_w_rel"] <= ROUTE_W_REL, rep
    assert max(rep["attn_rel"]) <= TOL_ATTN_REL, rep["attn_rel"]
    assert rep["h_abs"] <= TOL_H_ABS, rep
    assert rep["h_rel"] <= TOL_H_REL, rep
