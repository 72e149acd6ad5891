"""The vocab-sharded sweep on one GPU: a table split into G row ranges, each swept by
mtp_lm_head_shard_partial with its row offset and the global mask, the partials merged
by mtp_argmax_merge_partials. The argmax and its value must be bit-identical to the
unsharded sweep's, the log-probability within 2e-2 + 1e-2|ref| of the oracle's; then
ShardedLmHead over a one-rank NCCL group."""
import numpy as np
import pytest
import torch

from helpers import assert_close, to_dev, to_dev_u16
from mtp_speculative_draft_lm_b200 import _lib as L
from mtp_speculative_draft_lm_b200 import api, synth
from test_gpu_sweep import device_table, oracle_logprobs, oracle_quant, oracle_sweep

pytestmark = pytest.mark.gpu


def sharded(table, world, x, mask=None, words=0):
    M = x.shape[0]
    parts = torch.empty((world, M, 4), dtype=torch.float32, device="cuda")
    for r in range(world):
        off, cnt = api.shard_range(table.n, world, r)
        if cnt == 0:
            parts[r].zero_()
            parts[r, :, 0] = float("-inf")
            parts[r].view(torch.int32)[:, 1] = 2**31 - 1
            continue
        shard = api.table_rows(table, off, off + cnt)
        head = api.LmHead(shard)
        L.mtp_lm_head_shard_partial(shard.desc, cnt, off, x, M, mask, words,
                                    words if mask is not None else 0, parts[r], None,
                                    head.dev_err, head.ws, head.ws.numel())
        assert head.dev_err.item() == 0  # an empty shard is not an error
    idx = torch.empty((M,), dtype=torch.int32, device="cuda")
    val = torch.empty((M,), dtype=torch.float32, device="cuda")
    lp = torch.empty((M,), dtype=torch.float32, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    L.mtp_argmax_merge_partials(parts, world, M, idx, val, lp, err)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), val.cpu().numpy(), lp.cpu().numpy(), int(err.item())


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("world,M", [(1, 3), (2, 3), (3, 3), (8, 3), (3, 12), (2, 32)])
def test_shards_merge_to_the_whole_sweep(orc, fmt, world, M):
    n, k = 4133, {0: 256, 1: 512, 2: 1280}[fmt]
    w = synth.as_u16(synth.normal_bf16(synth._gen(70 + fmt), (n, k), 0.05))
    x = synth.as_u16(synth.normal_bf16(synth._gen(80 + world), (M, k), 1.0))
    q = oracle_quant(orc, w, fmt)
    table = device_table(q, fmt, n, k)
    xd = to_dev_u16(x)
    i0, v0, _, lp0 = api.LmHead(table).argmax(xd, logprob=True)
    idx, val, lp, err = sharded(table, world, xd)
    assert err == 0
    assert np.array_equal(idx, i0.cpu().numpy())
    assert np.array_equal(val.view(np.int32), v0.cpu().numpy().view(np.int32))
    ref_l, ref_i, _, _ = oracle_sweep(orc, q, fmt, k, x)
    assert np.array_equal(idx, ref_i)
    assert_close(lp, oracle_logprobs(orc, ref_l), "sharded log-probability")
    # a global mask: shards read their own tokens' bits; row 0 keeps only tokens of the
    # last shard, row 1 nothing at all
    words = (n + 31) // 32
    rng = np.random.default_rng(world)
    keep = rng.random((M, n)) < 0.1
    off_last, _ = api.shard_range(n, world, world - 1)
    keep[0, :off_last] = False
    keep[1] = False
    mask = synth.pack_mask(keep)
    md = to_dev(mask.reshape(-1))
    idx, val, lp, err = sharded(table, world, xd, md, words)
    i1, v1, _, lp1 = api.LmHead(table).argmax(xd, mask=md, mask_words=words,
                                              mask_stride_words=words, logprob=True)
    torch.cuda.synchronize()
    assert np.array_equal(idx, i1.cpu().numpy())
    assert np.array_equal(val.view(np.int32), v1.cpu().numpy().view(np.int32))
    assert idx[1] == 0 and val[1] == -np.inf and lp[1] == -np.inf
    assert err & L.MTP_DEVFLAG_EMPTY_MASK
    ref = oracle_logprobs(orc, ref_l, mask.reshape(-1), words, words)
    rest = [m for m in range(M) if m != 1]
    assert_close(lp[rest], ref[rest], "masked sharded log-probability")


def test_sharded_head_one_rank_nccl(orc):
    import torch.distributed as dist

    n, k, M = 2000, 512, 2
    w = synth.as_u16(synth.normal_bf16(synth._gen(90), (n, k), 0.05))
    x = synth.as_u16(synth.normal_bf16(synth._gen(91), (M, k), 1.0))
    table = api.bf16_table(to_dev_u16(w))
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        off, cnt = api.shard_range(n, 1, 0)
        head = api.ShardedLmHead(api.table_rows(table, off, off + cnt), off)
        idx, val, lp, err = head.argmax(to_dev_u16(x), logprob=True)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref_l, ref_i, _, _ = orc.lm_head_argmax(0, w, k, x)
    assert np.array_equal(idx.cpu().numpy(), ref_i) and err.item() == 0
    assert_close(lp.cpu().numpy(), oracle_logprobs(orc, ref_l), "log-probability")
