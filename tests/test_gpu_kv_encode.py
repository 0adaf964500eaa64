"""The GPU's fp8 e4m3 encoder -- the conversion the step uses to write its
keys and values into the cache, exported as msk_kv_encode -- against the
oracle's encoder, bit for bit, on fixed fp32 inputs: every finite e4m3 value,
every rounding midpoint (ties go to the even code) and its fp32 neighbours,
subnormals, signed zeros, values beyond 448 (saturated), infinities and NaN
(the fp8 KV cache of the pages, "Key points"; the format is OFP8 E4M3)."""
import numpy as np
import pytest
import torch

import oracle
import verify_step_megakernel_b200 as msk

pytestmark = pytest.mark.gpu


def _grid():
    return torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()  # 0 .. 448


def _inputs():
    g = _grid()
    mids = 0.5 * (g[:-1] + g[1:])  # exact in fp32
    m32 = mids.astype(np.float32)
    assert np.array_equal(m32.astype(np.float64), mids)
    up = np.nextafter(m32, np.float32(np.inf))
    dn = np.nextafter(m32, np.float32(0))
    big = np.array([448.0, 448.5, 449.0, 463.99, 464.0, 464.01, 479.0, 480.0, 500.0, 1e6, 3.0e38], np.float32)
    tiny = np.array([2.0 ** -10, np.nextafter(np.float32(2.0 ** -10), np.float32(1)), 2.0 ** -11, 1e-30, 1e-45,
                     2.0 ** -9, 2.0 ** -6, np.nextafter(np.float32(2.0 ** -6), np.float32(0))], np.float32)
    pos = np.concatenate([g.astype(np.float32), m32, up, dn, big, tiny])
    x = np.concatenate([pos, -pos, np.array([0.0, -0.0, np.inf, -np.inf], np.float32)])
    rng = np.random.default_rng(9)
    x = np.concatenate([x, (rng.standard_normal(4093) * 3).astype(np.float32)])  # a ragged tail
    return x.astype(np.float32)


def test_kv_encoder_matches_oracle_bit_exactly():
    x = _inputs()
    dev = torch.device("cuda", 0)
    xin = torch.from_numpy(x).to(dev)
    out = torch.full((x.size,), 0x55, dtype=torch.uint8, device=dev)
    msk.msk_kv_encode(xin.data_ptr(), out.data_ptr(), x.size)
    torch.cuda.synchronize(dev)
    got = out.cpu().numpy()
    want = oracle.e4m3_encode(x.astype(np.float64))
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, [(float(x[i]), int(got[i]), int(want[i])) for i in bad[:10]]
    # the ties really were exercised: both parities of the lower neighbour
    g = _grid()
    lo_codes = np.arange(126)
    tie = oracle.e4m3_encode(0.5 * (g[:-1] + g[1:]))
    assert np.array_equal(tie, np.where(lo_codes % 2 == 0, lo_codes, lo_codes + 1))


def test_kv_encoder_nan_and_empty():
    dev = torch.device("cuda", 0)
    x = torch.tensor([float("nan"), -float("nan"), 1.0, 2.0], dtype=torch.float32, device=dev)
    out = torch.zeros(4, dtype=torch.uint8, device=dev)
    msk.msk_kv_encode(x.data_ptr(), out.data_ptr(), 4)
    torch.cuda.synchronize(dev)
    o = out.cpu().numpy()
    assert (o[0] & 0x7F) == 0x7F and (o[1] & 0x7F) == 0x7F and o[2] == 0x38 and o[3] == 0x40
    msk.msk_kv_encode(0, 0, 0)  # nothing to do
    with pytest.raises(msk.MskError) as e:
        msk.msk_kv_encode(x.data_ptr() + 4, out.data_ptr(), 3)  # misaligned input
    assert e.value.code == 1
