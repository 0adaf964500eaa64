"""A device wait that runs out ends the step with MSK_ERR_TIMEOUT, records
where, and leaves the handle usable.

The library's test hook (msk_debug_t.hold_barrier) makes CTA 0 withhold its
arrival at one grid barrier of the step, so every CTA's bounded wait there
gives up after the handle's wait_timeout_us (20 ms here).  Nothing traps or
faults: the CTAs let their copies in flight land, free their tensor memory
and return.  The next step on the same handle, with the hook off, must pass
parity against the oracle."""
import pytest
import torch

import synth
import synth.gpu as sg
import verify_step_megakernel_b200 as msk
from synth.engine import Engine
from tests._parity import assert_parity, run_parity

pytestmark = pytest.mark.gpu

TIMEOUT = 7
# grid barriers of a step: 1 after the input norm, then per layer l the
# barriers closing phases 1 (QKV) .. 7 (router), 9 (gate/up), 10 (down) and
# 11 (combine): barrier n = 2 + 10 l + index in this list
PHASES_WITH_BARRIER = [1, 2, 3, 4, 5, 6, 7, 9, 10, 11]


def _site(n):
    if n == 1:
        return 0, 0
    l, i = divmod(n - 2, 10)
    return l, PHASES_WITH_BARRIER[i]


def _held_step(eng, hid, pos, n):
    w, dev = eng.w, eng.dev
    msk.msk_set_debug(eng.h, hold_barrier=n)
    out = torch.empty((w.T, w.d_model), dtype=torch.int16, device=dev)
    p = torch.tensor(pos, dtype=torch.int32, device=dev)
    msk.msk_step(eng.h, hid.data_ptr(), p.data_ptr(), w.n_seqs, w.tokens_per_seq, eng.kv, out.data_ptr(),
                 torch.cuda.current_stream(dev).cuda_stream)
    torch.cuda.synchronize(dev)
    msk.msk_set_debug(eng.h)
    return msk.msk_step_status_at(eng.h)


@pytest.mark.parametrize("tau", [msk.TAU_NEVER, 1], ids=["cuda_core", "tensor_core"])
def test_withheld_barrier_times_out_and_the_next_step_is_exact(tau):
    w = synth.WORKLOADS["tiny"]
    eng = Engine(w, timeout_us=20000, tau=tau)
    try:
        eng.fill_past()
        hid = sg.hidden(w)
        pos = w.positions()
        # barriers with different work in flight when the wait starts: after
        # the input norm, after attention (W_o tiles issued), after gate/up
        # (down tiles pending), and in layer 1 after QK-norm
        for n in (1, 5, 10, 14):
            st, layer, phase, cta = _held_step(eng, hid, pos, n)
            assert st == TIMEOUT and (layer, phase) == _site(n), (n, st, layer, phase, cta)
            assert 0 <= cta < 148
            assert msk.msk_step_status_at(eng.h)[0] == 0  # read once, then cleared
        # the hook off: the next step is the ordinary one, at parity
        rep, _, _ = run_parity(w, eng, hid, pos)
        assert_parity(rep)
    finally:
        eng.close()
