"""The vocab-sharded sweep's host side on CPU: shard ranges, and the exchange of the
16-byte partials between two gloo ranks, with each rank's partial computed by the
oracle on its own rows; the merged result must equal the oracle on the whole table."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from mtp_speculative_draft_lm_b200 import api, synth


@pytest.mark.parametrize("n,world", [(154880, 8), (100, 3), (20, 4), (16, 1), (4133, 7)])
def test_shard_ranges_tile_the_table(n, world):
    covered = 0
    for r in range(world):
        off, cnt = api.shard_range(n, world, r)
        assert off == covered and cnt >= 0
        if cnt and off + cnt < n:
            assert cnt % 16 == 0
        covered += cnt
    assert covered == n


def oracle_partial(orc, w, k, x, r0, r1, mask=None, words=0):
    """A shard's partial from the oracle: the shard's argmax (global row), its maximum,
    and exp(-log-probability) = sum over its allowed rows of exp(l - max)."""
    M = x.shape[0]
    out = np.zeros((M, 4), np.float32)
    if r1 <= r0:
        out[:, 0] = -np.inf
        out.view(np.int32)[:, 1] = np.iinfo(np.int32).max
        return out
    lg, _, _, _ = orc.lm_head_argmax(0, w[r0:r1], k, x)
    for m in range(M):
        allowed = np.ones(r1 - r0, bool)
        if mask is not None:
            t = np.arange(r0, r1)
            words_m = mask[m].view(np.uint32)
            allowed = ((words_m[t // 32] >> (t % 32).astype(np.uint32)) & 1).astype(bool)
        if not allowed.any():
            out[m, 0] = -np.inf
            out.view(np.int32)[m, 1] = np.iinfo(np.int32).max
            continue
        l = np.where(allowed, lg[m], -np.inf)
        i = int(np.argmax(l))
        out[m, 0] = l[i]
        out.view(np.int32)[m, 1] = r0 + i
        out[m, 2] = np.exp(-orc.top1_logprob(l))
    return out


def merge(parts):
    """Plain merge of [world, M, 4] partials: largest maximum, lowest row on ties."""
    world, M, _ = parts.shape
    idx, val = [], []
    for m in range(M):
        best = (-np.inf, np.iinfo(np.int32).max)
        for r in range(world):
            v, i = float(parts[r, m, 0]), int(parts[r, m].view(np.int32)[1])
            if i != np.iinfo(np.int32).max and (v > best[0] or (v == best[0] and i < best[1])):
                best = (v, i)
        val.append(best[0])
        idx.append(best[1])
    return np.array(idx), np.array(val)


def _rank(rank, world, port, q):
    import torch.distributed as dist

    import oracle as orc  # built by the parent

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        n, k, M = 300, 128, 3
        w = synth.as_u16(synth.normal_bf16(synth._gen(7), (n, k), 0.05))
        x = synth.as_u16(synth.normal_bf16(synth._gen(8), (M, k), 1.0))
        r0, cnt = api.shard_range(n, world, rank)
        local = torch.from_numpy(oracle_partial(orc, w, k, x, r0, r0 + cnt))
        parts = api.exchange_partials(local).numpy()
        q.put((rank, parts))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_gloo_two_ranks_exchange_matches_whole_table(orc):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank holds the same gathered partials, rank-major
    assert np.array_equal(got[0], got[1])
    n, k, M = 300, 128, 3
    w = synth.as_u16(synth.normal_bf16(synth._gen(7), (n, k), 0.05))
    x = synth.as_u16(synth.normal_bf16(synth._gen(8), (M, k), 1.0))
    for r in range(world):
        r0, cnt = api.shard_range(n, world, r)
        assert np.array_equal(got[0][r], oracle_partial(orc, w, k, x, r0, r0 + cnt))
    idx, val = merge(got[0])
    ref_l, ref_i, ref_v, _ = orc.lm_head_argmax(0, w, k, x)
    assert np.array_equal(idx, ref_i)
    assert np.allclose(val, ref_v.astype(np.float32))
