"""The allocation-free sweep entry point (mtp_lm_head_argmax_noalloc).

It serves callers that cannot allocate device memory when they run a draft: they
pass inputs and outputs, and the sweep's scratch comes from a static array inside
the library. This checks, through the C ABI, that two calls in a row give the same
results as mtp_lm_head_argmax with a caller workspace, within the parity tolerance
the other tests use (2e-2 + 1e-2 |ref| on values and logits; the same argmax index).
The file sorts last so that a failure here stops a `-x` run after everything else.
"""
import numpy as np
import pytest
import torch

from mtp_speculative_draft_lm_b200 import _lib as L
from mtp_speculative_draft_lm_b200 import api, synth

pytestmark = pytest.mark.gpu

TOL_ABS, TOL_REL = 2e-2, 1e-2


def close(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return bool(np.all(np.abs(a - b) <= TOL_ABS + TOL_REL * np.abs(b)))


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_noalloc_matches_workspace_entry_point(fmt):
    n, k, M = 5000, 1024, 3
    d = synth.head_table(21 + fmt, n, k, M)
    w = d["W"].cuda()
    table = api.bf16_table(w) if fmt == 0 else (api.quantize_fp8(w) if fmt == 1 else
                                                 api.quantize_nvfp4(w))
    x = d["x"].cuda()
    head = api.LmHead(table)
    ref_idx, ref_val, ref_lg = head.argmax(x, logits=True)
    torch.cuda.synchronize()
    assert L.mtp_noalloc_scratch_bytes() >= L.mtp_lm_head_ws_bytes(table.desc, n, M)
    for _ in range(2):
        idx = torch.full((M,), -7, dtype=torch.int32, device="cuda")
        val = torch.zeros((M,), dtype=torch.float32, device="cuda")
        lg = torch.zeros((M, n), dtype=torch.bfloat16, device="cuda")
        err = torch.zeros((1,), dtype=torch.int32, device="cuda")
        L.mtp_lm_head_argmax_noalloc(table.desc, n, x, M, None, 0, 0, idx, val, lg, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert np.array_equal(idx.cpu().numpy(), ref_idx.cpu().numpy())
        assert np.array_equal(idx.cpu().numpy(), d["top"])
        assert close(val.cpu().numpy(), ref_val.cpu().numpy())
        assert close(lg.float().cpu().numpy(), ref_lg.float().cpu().numpy())


def test_noalloc_masked_rows_and_rejects():
    n, k, M = 3000, 512, 2
    d = synth.head_table(31, n, k, M, mask_keep=0.1)
    table = api.bf16_table(d["W"].cuda())
    x = d["x"].cuda()
    words = d["mask"].shape[1]
    mask = torch.from_numpy(d["mask"].reshape(-1)).cuda()
    for _ in range(2):
        idx = torch.empty((M,), dtype=torch.int32, device="cuda")
        L.mtp_lm_head_argmax_noalloc(table.desc, n, x, M, mask, words, words, idx, None, None,
                                     None)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), d["second"])
    bad = L.raw_status("mtp_lm_head_argmax_noalloc", None, n, x.data_ptr(), M, None, 0, 0,
                       idx.data_ptr(), None, None, None, None)
    assert bad == L.MTP_ERR_INVALID_ARG
