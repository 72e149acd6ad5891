"""Failure handling on the GPU without a fault: a pipeline wait that can never complete
gives up after its limit, reports MTP_DEVFLAG_TIMEOUT through the device error word and
lets the kernel end, and the context stays usable (mtp_debug_wait_timeout runs the
pipelines' own wait helpers with a short limit)."""
import time

import numpy as np
import pytest
import torch

from mtp_speculative_draft_lm_b200 import _lib as L
from mtp_speculative_draft_lm_b200 import api, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [0, 1], ids=["mbarrier", "counter"])
def test_bounded_wait_times_out_and_reports(which):
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    ctr = torch.zeros((1,), dtype=torch.int32, device="cuda")  # nothing ever increments it
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    L.mtp_debug_wait_timeout(which, 2_000_000, ctr, err)  # about a millisecond of SM clock
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert int(err.item()) == L.MTP_DEVFLAG_TIMEOUT
    assert L.mtp_devflags_status(int(err.item())) == L.MTP_ERR_INVALID_ARG
    # the context is still usable
    d = synth.head_table(5, 700, 256, 2)
    idx, _, _ = api.LmHead(api.bf16_table(d["W"].cuda())).argmax(d["x"].cuda())
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), d["top"])
