"""The device fill of the input generator equals the host fill, bit for bit
(so the oracle, which regenerates on the host, sees the GPU's inputs)."""
import numpy as np
import pytest
import torch

import synth
import synth.gpu as sg

pytestmark = pytest.mark.gpu


def test_device_fill_equals_host_fill():
    w = synth.WORKLOADS["dec8"]
    wts = sg.DeviceWeights(w.with_(n_layers=2, sliding=[1, 0]))
    for role in ("wq", "wk", "wo"):
        c, s, gs = wts.layers[1][role]
        hc, hs, hgs = synth.host_nvfp4(w, role, 1)
        dc = torch.empty(hc.size, dtype=torch.uint8, device="cuda")
        ds = torch.empty(hs.size, dtype=torch.uint8, device="cuda")
        synth.dev_nvfp4(w, role, 1, 0, dc.data_ptr(), ds.data_ptr())
        torch.cuda.synchronize()
        assert np.array_equal(dc.cpu().numpy(), hc.ravel()) and np.array_equal(ds.cpu().numpy(), hs.ravel())
        assert gs == hgs
    # one expert of each expert tensor, from the stacked device copy
    # (the stacked tensors are filled by one launch per role)
    for role in ("w_gate", "w_up", "w_down"):
        c, s, gs = wts.layers[0][role]
        dev_c = wts.keep[[i for i, t in enumerate(wts.keep) if t.data_ptr() == c][0]]
        dev_s = wts.keep[[i for i, t in enumerate(wts.keep) if t.data_ptr() == s][0]]
        for e in (0, 201, w.n_experts - 1):
            hc, hs, hgs = synth.host_nvfp4(w, role, 0, e)
            assert np.array_equal(dev_c[e * hc.size:(e + 1) * hc.size].cpu().numpy(), hc.ravel())
            assert np.array_equal(dev_s[e * hs.size:(e + 1) * hs.size].cpu().numpy(), hs.ravel())
            assert gs == hgs
    for name in ("router", "q_norm_g", "moe_norm_g"):
        ptr = wts.layers[1][name]
        host = synth.host_vec(w, name, 1).ravel()
        dev_t = [t for t in wts.keep if t.data_ptr() == ptr][0]
        assert np.array_equal(dev_t.cpu().numpy(), host)
    hid = sg.hidden(w.with_(n_seqs=3, tokens_per_seq=5))
    assert np.array_equal(hid.cpu().numpy().view(np.uint16), synth.host_hidden(w, 3, 5))
    kb = torch.empty((777, w.n_kv_heads * w.head_dim), dtype=torch.uint8, device="cuda")
    vb = torch.empty_like(kb)
    sg.past_chunk(w, 5, 0, 12345, 777, kb, vb)
    torch.cuda.synchronize()
    for h in range(w.n_kv_heads):
        hk, hv = synth.host_past(w, 5, 0, h, 12345, 777)
        assert np.array_equal(kb.cpu().numpy()[:, h * 128:(h + 1) * 128], hk)
        assert np.array_equal(vb.cpu().numpy()[:, h * 128:(h + 1) * 128], hv)
