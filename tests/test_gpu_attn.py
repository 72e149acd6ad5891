"""Single-token paged decode attention over the E4M3 KV cache on the GPU against the
oracle: random caches at several head widths, group sizes, lengths (one row, ragged
tails, many 256-row pieces), scales, a missing block, and the cache the prefill writes
for a whole prompt. Outputs are bf16 of an fp32 softmax: within 2e-2 + 1e-2|ref|."""
import numpy as np
import pytest
import torch

from helpers import assert_close, bf16_bits_to_f64, to_dev, to_dev_u16, u16_of
from mtp_speculative_draft_lm_b200 import _lib as L
from mtp_speculative_draft_lm_b200 import api, synth

pytestmark = pytest.mark.gpu


def case(orc, seed, nq, nkv, hd, seq, bs=16, extra=3):
    rng = np.random.default_rng(seed)
    nb = seq // bs + 1 + extra
    bt = rng.permutation(nb).astype(np.int32)
    kc = orc.e4m3_encode(rng.normal(0, 1, nb * bs * nkv * hd)).reshape(nb, bs, nkv, hd)
    vc = orc.e4m3_encode(rng.normal(0, 1, nb * bs * nkv * hd)).reshape(nb, bs, nkv, hd)
    q = orc.f64_to_bf16(rng.normal(0, 1, (nq, hd)))
    return q, kc, vc, bt, nb


def run(q, nkv, kc, vc, bt, seq, **kw):
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    out, _ = api.paged_decode_attn(to_dev_u16(q), nkv, to_dev(kc), to_dev(vc), to_dev(bt), seq,
                                   dev_err=err, **kw)
    torch.cuda.synchronize()
    return bf16_bits_to_f64(u16_of(out)), int(err.item())


@pytest.mark.parametrize("nq,nkv,hd,seq", [(8, 8, 128, 1), (64, 8, 128, 300), (16, 2, 64, 257),
                                           (4, 1, 256, 1000), (32, 2, 128, 4097)])
def test_attention_matches_oracle(orc, nq, nkv, hd, seq):
    q, kc, vc, bt, nb = case(orc, nq + hd + seq, nq, nkv, hd, seq)
    got, err = run(q, nkv, kc, vc, bt, seq)
    assert err == 0
    ref, flags = orc.paged_decode_attn(q, nkv, kc, vc, bt, 16, nb, seq)
    assert flags == 0
    assert_close(got, ref, "attention output")


def test_attention_scales_and_missing_block(orc):
    q, kc, vc, bt, nb = case(orc, 7, 8, 2, 128, 100)
    got, err = run(q, 2, kc, vc, bt, 100, k_scale=0.5, v_scale=2.0, scale=0.3)
    ref, _ = orc.paged_decode_attn(q, 2, kc, vc, bt, 16, nb, 100, k_scale=0.5, v_scale=2.0, scale=0.3)
    assert err == 0
    assert_close(got, ref, "scaled")
    got, err = run(q, 2, kc, vc, bt[:3], 100)  # rows 48.. have no block: skipped and flagged
    ref, flags = orc.paged_decode_attn(q, 2, kc, vc, bt[:3], 16, nb, 100)
    assert err == L.MTP_DEVFLAG_BAD_SLOT and flags & orc.FLAG_BAD_SLOT
    assert_close(got, ref, "missing block")


def test_attention_over_the_prefill_cache(orc):
    """Decode attention of a random query over the cache mtp_prefill_kv writes for a
    1,000-row prompt (hidden 512, 4 KV heads x 128), against the oracle on the same bytes."""
    d = synth.prefill_inputs(seed=84, R=1000, vocab=700, h=512, nkv=4, hd=128)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    nb = int(d["num_blocks"])
    kc = torch.zeros((nb, 16, 4, 128), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    api.prefill_kv(dev, kc, vc, chunk_rows=256)
    torch.cuda.synchronize()
    rng = np.random.default_rng(2)
    q = orc.f64_to_bf16(rng.normal(0, 1, (16, 128)))
    kcn, vcn, bt = kc.cpu().numpy(), vc.cpu().numpy(), d["block_table"].numpy()
    got, err = run(q, 4, kcn, vcn, bt, 1000)
    ref, _ = orc.paged_decode_attn(q, 4, kcn, vcn, bt, 16, nb, 1000)
    assert err == 0
    assert_close(got, ref, "prefill cache")


@pytest.mark.parametrize("bs,seq", [(32, 777), (64, 1000), (8, 333)])
def test_attention_block_sizes(orc, bs, seq):
    """Blocks of 32 and 64 rows (several 16-row copies inside one block) and of 8 rows (the
    16-byte copy path)."""
    q, kc, vc, bt, nb = case(orc, 11 + bs, 16, 2, 128, seq, bs=bs)
    got, err = run(q, 2, kc, vc, bt, seq)
    ref, flags = orc.paged_decode_attn(q, 2, kc, vc, bt, bs, nb, seq)
    assert err == 0 and flags == 0
    assert_close(got, ref, f"block size {bs}")


def test_attention_nan_past_the_end(orc):
    """Rows past the sequence inside its last block hold the E4M3 NaN code in K and V: they
    are never read (a finite output equal to the oracle's, which reads rows < seq_len)."""
    seq = 70  # the last block holds rows 64 .. 69 of the sequence and 10 more
    q, kc, vc, bt, nb = case(orc, 5, 16, 2, 128, seq)
    for pos in range(seq, (seq // 16 + 1) * 16):
        kc[bt[pos // 16], pos % 16] = 0x7F
        vc[bt[pos // 16], pos % 16] = 0x7F
    got, err = run(q, 2, kc, vc, bt, seq)
    ref, _ = orc.paged_decode_attn(q, 2, kc, vc, bt, 16, nb, seq)
    assert err == 0
    assert np.all(np.isfinite(got))
    assert_close(got, ref, "NaN rows past the end")


def test_attention_unaligned_query(orc):
    """q only 2-byte aligned (a view one element into a buffer): the per-head staging."""
    q, kc, vc, bt, nb = case(orc, 9, 16, 2, 128, 300)
    buf = torch.empty((q.size + 1,), dtype=torch.bfloat16, device="cuda")
    buf[1:] = to_dev_u16(q).reshape(-1)
    qd = buf[1:].reshape(q.shape)
    assert qd.data_ptr() % 16 == 2
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    out, _ = api.paged_decode_attn(qd, 2, to_dev(kc), to_dev(vc), to_dev(bt), 300, dev_err=err)
    torch.cuda.synchronize()
    ref, _ = orc.paged_decode_attn(q, 2, kc, vc, bt, 16, nb, 300)
    assert int(err.item()) == 0
    assert_close(bf16_bits_to_f64(u16_of(out)), ref, "unaligned q")
