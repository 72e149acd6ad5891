"""Device encoders (E4M3, E2M1) against the oracle on every bf16 value, every
midpoint +-1 ulp and a dense grid: bit-exact."""
import numpy as np
import pytest
import torch

from helpers import to_dev
from mtp_speculative_draft_lm_b200 import _lib as L

pytestmark = pytest.mark.gpu


def e4m3_mags(orc):
    return orc.e4m3_value(np.arange(127))


def inputs_e4m3(orc):
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    f = f[~np.isnan(f)]
    mags = e4m3_mags(orc)
    mids = ((mags[1:] + mags[:-1]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)),
                           np.nextafter(mids, np.float32(-np.inf))])
    rng = np.random.default_rng(0)
    rnd = (rng.standard_normal(200000) * np.exp2(rng.integers(-20, 12, 200000))).astype(np.float32)
    return np.concatenate([f, near, -near, rnd]).astype(np.float32)


def run(fn, v):
    inp = to_dev(v)
    out = torch.empty(v.shape, dtype=torch.uint8, device="cuda")
    fn(inp, v.size, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_e4m3_encoder_bit_exact(orc):
    v = inputs_e4m3(orc)
    got = run(L.mtp_debug_encode_e4m3, v)
    ref = orc.e4m3_encode(v.astype(np.float64))
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (v[bad[:8]], got[bad[:8]], ref[bad[:8]])


def test_e2m1_encoder_bit_exact(orc):
    grid = (np.arange(-8 * 8192, 8 * 8192 + 1) / 8192.0).astype(np.float32)
    mags = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    mids = (mags[1:] + mags[:-1]) / 2
    near = np.concatenate([mids, np.nextafter(mids, np.float32(9)), np.nextafter(mids, np.float32(-1))])
    v = np.concatenate([grid, near, -near, np.array([-0.0, 0.0, 1e30, -1e30], np.float32)])
    got = run(L.mtp_debug_encode_e2m1, v)
    ref = orc.e2m1_encode(v.astype(np.float64))
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (v[bad[:8]], got[bad[:8]], ref[bad[:8]])
