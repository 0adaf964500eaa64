"""msk_step_static: the step with its working memory in the library's fixed
array (no allocation) gives the results of msk_step, bit for bit (the same
deterministic kernel: every reduction runs in a fixed order).

Collected last on purpose: it must pass on its own and after every other
GPU test has used the library on the same device."""
import numpy as np
import pytest
import torch

import synth.gpu as sg
import verify_step_megakernel_b200 as msk
from synth.configs import WORKLOADS
from synth.engine import Engine, config_struct



@pytest.mark.gpu
def test_static_step_matches_step_twice():
    # 2 sequences x 8 draft tokens of the 8-layer d_model 2048 model
    # (working memory about 6.7 MiB of the 8 MiB array), 4096 past tokens
    w = WORKLOADS["ver8"].with_(past=4096)
    eng = Engine(w)
    try:
        eng.fill_past()
        dev = eng.dev
        hidden = sg.hidden(w, eng.device)
        pos = torch.tensor(w.positions(), dtype=torch.int32, device=dev)
        S, Tq = pos.shape
        stream = torch.cuda.current_stream(dev).cuda_stream
        msk.msk_set_debug(eng.h)

        ref = torch.empty((S * Tq, w.d_model), dtype=torch.int16, device=dev)
        msk.msk_step(eng.h, hidden.data_ptr(), pos.data_ptr(), S, Tq, eng.kv, ref.data_ptr(), stream)
        torch.cuda.synchronize(dev)
        assert msk.msk_step_status(eng.h) == 0
        ref_np = ref.cpu().numpy().view(np.uint16)

        # two calls in a row, same positions: each rewrites the step's own KV
        # rows with the same values, so both must reproduce the reference
        for call in range(2):
            out = torch.full((S * Tq, w.d_model), -1, dtype=torch.int16, device=dev)
            msk.msk_step_static(eng.h, hidden.data_ptr(), pos.data_ptr(), S, Tq, eng.kv, out.data_ptr(), stream)
            torch.cuda.synchronize(dev)
            assert msk.msk_step_status(eng.h) == 0, f"call {call}"
            out_np = out.cpu().numpy().view(np.uint16)
            assert np.array_equal(out_np, ref_np), (call, int((out_np != ref_np).sum()))
            st = msk.msk_query(eng.h)
            assert st.n_layers == w.n_layers and st.algorithmic_bytes > 0
    finally:
        eng.close()


@pytest.mark.gpu
def test_static_step_rejects_shapes_beyond_the_array():
    # 16 x 4 tokens of d_model 4096 need about 17.7 MiB of working memory:
    # refused before any device work.  msk_create reads the expert weights
    # (it repacks them into its own tiles), so they are real buffers of the
    # right sizes (zeros), on a model with few small experts.
    w = WORKLOADS["large"].with_(n_layers=1, sliding=[1], n_experts=32, expert_dim=128)
    dev = torch.device("cuda", 0)
    d, hd, E, f = w.d_model, w.head_dim, w.n_experts, w.expert_dim
    qd, kvd = w.n_q_heads * hd, w.n_kv_heads * hd
    keep = []

    def nv(rows, K):
        c = torch.zeros(rows * K // 2, dtype=torch.uint8, device=dev)
        s = torch.zeros(rows * K // 16, dtype=torch.uint8, device=dev)
        keep.extend([c, s])
        return msk.Nvfp4(c.data_ptr(), s.data_ptr(), 1.0)

    ones_d = torch.ones(d, dtype=torch.float32, device=dev)
    ones_hd = torch.ones(hd, dtype=torch.float32, device=dev)
    router = torch.zeros((E, d), dtype=torch.float32, device=dev)
    lw = msk.LayerWeights()
    lw.attn_norm_g = lw.moe_norm_g = ones_d.data_ptr()
    lw.q_norm_g = lw.k_norm_g = ones_hd.data_ptr()
    lw.router = router.data_ptr()
    lw.wq, lw.wk, lw.wv, lw.wo = nv(qd, d), nv(kvd, d), nv(kvd, d), nv(d, qd)
    lw.w_gate, lw.w_up, lw.w_down = nv(E * f, d), nv(E * f, d), nv(E * d, f)
    h = msk.msk_create(config_struct(w), [lw], 0)
    kv = msk.msk_kv_create(h, w.n_seqs, 16)
    try:
        hid = torch.zeros((w.T, d), dtype=torch.int16, device=dev)
        out = torch.zeros_like(hid)
        pos = torch.zeros((w.n_seqs, w.tokens_per_seq), dtype=torch.int32, device=dev)
        with pytest.raises(msk.MskError) as ei:
            msk.msk_step_static(h, hid.data_ptr(), pos.data_ptr(), w.n_seqs, w.tokens_per_seq, kv, out.data_ptr())
        assert ei.value.code == 2  # MSK_ERR_UNSUPPORTED
        assert msk.msk_query(h).scratch_bytes > msk.STATIC_SCRATCH_BYTES
    finally:
        msk.msk_kv_destroy(kv)
        msk.msk_destroy(h)
