"""Quantizers on the GPU against the oracle: codes, block scales, row and global
scales bit-exact, from a few rows to the benchmark tables (154,880 x 4,096 FP8;
131,072 x 5,120 NVFP4)."""
import os

import numpy as np
import pytest
import torch

from helpers import to_dev_u16
from mtp_speculative_draft_lm_b200 import api, synth

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def small_table(seed, n, k, std=0.02):
    w = synth.as_u16(synth.normal_bf16(synth._gen(seed), (n, k), std))
    w = w.copy()
    w[min(3, n - 1)] = 0                     # an all-zero row
    w[0, : min(16, k)] = 0x8000             # negative zeros
    return w


@pytest.mark.parametrize("n,k", [(1, 16), (37, 48), (1000, 4096), (333, 5120)])
def test_fp8_quantizer_bit_exact(orc, n, k):
    w = small_table(100 + n, n, k)
    t = api.quantize_fp8(to_dev_u16(w))
    torch.cuda.synchronize()
    codes, scale = orc.quantize_fp8(w)
    assert np.array_equal(t.row_scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(t.data.cpu().numpy(), codes)


@pytest.mark.parametrize("n,k", [(1, 32), (37, 64), (1000, 4096), (129, 5120), (50, 1056)])
def test_nvfp4_quantizer_bit_exact(orc, n, k):
    w = small_table(200 + n, n, k)
    t = api.quantize_nvfp4(to_dev_u16(w))
    torch.cuda.synchronize()
    codes, bscale, g = orc.quantize_nvfp4(w)
    assert np.float32(t.global_scale.item()).view(np.uint32) == np.float32(g).view(np.uint32)
    bs = t.block_scale.cpu().numpy()
    assert np.array_equal(bs[:, : k // 16], bscale)
    assert np.all(bs[:, k // 16:] == 0)
    assert np.array_equal(t.data.cpu().numpy(), codes)


def test_nvfp4_quantizer_golden_block():
    vals = {}
    for line in open(os.path.join(GOLDEN, "nvfp4_block.txt")):
        if ":" in line and not line.startswith("#"):
            key, rest = line.split(":", 1)
            vals[key.strip()] = rest.split()
    x = np.array([float(v) for v in vals["values"]] + [0.0] * 16, np.float32)
    w = torch.tensor(x).to(torch.bfloat16).view(1, 64).cuda()
    t = api.quantize_nvfp4(w)
    torch.cuda.synchronize()
    assert t.global_scale.item() == float(vals["global_scale"][0])
    assert list(t.block_scale.cpu().numpy()[0]) == [int(v, 16) for v in vals["block_scales"]] + [0] * 13
    assert list(t.data.cpu().numpy()[0]) == [int(v, 16) for v in vals["codes"]] + [0] * 8


def test_quantizer_workspace_is_reusable(orc):
    w = small_table(7, 64, 256)
    ws = torch.zeros((api.L.mtp_quantize_nvfp4_ws_bytes(64, 256),), dtype=torch.uint8,
                     device="cuda")
    a = api.quantize_nvfp4(to_dev_u16(w), ws=ws)
    b = api.quantize_nvfp4(to_dev_u16(w * 0 + w), ws=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert torch.equal(a.data, b.data) and torch.equal(a.block_scale, b.block_scale)


def test_fp8_quantizer_full_table(orc):
    cfg = synth.FP8_HEAD
    d = synth.head_table(cfg["seed"], cfg["N"], cfg["K"], max(cfg["Ms"]))
    w = synth.as_u16(d["W"])
    t = api.quantize_fp8(d["W"].cuda())
    torch.cuda.synchronize()
    codes, scale = orc.quantize_fp8(w)
    assert np.array_equal(t.row_scale.cpu().numpy().view(np.uint32), scale.view(np.uint32))
    assert np.array_equal(t.data.cpu().numpy(), codes)


def test_nvfp4_quantizer_full_table(orc):
    cfg = synth.NVFP4_HEAD
    d = synth.head_table(cfg["seed"], cfg["N"], cfg["K"], max(cfg["Ms"]))
    w = synth.as_u16(d["W"])
    t = api.quantize_nvfp4(d["W"].cuda())
    torch.cuda.synchronize()
    codes, bscale, g = orc.quantize_nvfp4(w)
    assert np.float32(t.global_scale.item()) == np.float32(g)
    assert np.array_equal(t.block_scale.cpu().numpy()[:, : cfg["K"] // 16], bscale)
    assert np.array_equal(t.data.cpu().numpy(), codes)
