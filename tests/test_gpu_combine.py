"""The combiner (embedding row, two RMSNorms, concat, fc) and the tiny end-to-end
draft step (hidden 256, vocab 4096) on the GPU against the oracle."""
import numpy as np
import pytest
import torch

from helpers import (assert_argmax, assert_close, bf16_bits_to_f64, pad_scales, to_dev,
                     to_dev_u16, u16_of)
from mtp_speculative_draft_lm_b200 import _lib as L
from mtp_speculative_draft_lm_b200 import api, synth

pytestmark = pytest.mark.gpu


def draft(M, seed=synth.TINY["seed"], h=synth.TINY["h"], vocab=synth.TINY["vocab"]):
    d = synth.tiny_draft(seed=seed, vocab=vocab, h=h, M=M)
    return {k: (synth.as_u16(v) if isinstance(v, torch.Tensor) and v.dtype == torch.bfloat16
                else v) for k, v in d.items()}


def gpu_combine(d, fc_table=None, tokens=None, norm_mode=0):
    fc = fc_table or api.bf16_table(to_dev_u16(d["fc"]))
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    tok = to_dev(np.asarray(d["tokens"] if tokens is None else tokens, np.int32))
    y = api.combine(to_dev_u16(d["embed"]), tok, to_dev_u16(d["hidden"]),
                    to_dev_u16(d["w_norm_embed"]), to_dev_u16(d["w_norm_hidden"]), d["eps"], fc,
                    dev_err=err, norm_mode=norm_mode)
    torch.cuda.synchronize()
    return u16_of(y), int(err.item())


@pytest.mark.parametrize("M", [1, 2, 5, 8, 16])
def test_combine_matches_oracle(orc, M):
    d = draft(M)
    y, err = gpu_combine(d)
    ref, _, flags = orc.combine(d["embed"], d["tokens"].numpy(), d["hidden"], d["w_norm_embed"],
                                d["w_norm_hidden"], d["eps"], d["fc"])
    assert err == 0 and flags == 0
    assert_close(bf16_bits_to_f64(y), bf16_bits_to_f64(ref), "y")
    # bf16 outputs: all but a handful identical, none more than one bf16 ulp apart
    diff = np.abs(y.astype(np.int32) - ref.astype(np.int32))
    assert diff.max() <= 1 and (diff > 0).mean() < 0.02


@pytest.mark.parametrize("M", [1, 7])
def test_combine_one_plus_w(orc, M):
    """norm_mode 1: every norm weight is 1 + w; the plain mode's output must differ."""
    d = draft(M, seed=77)
    y, err = gpu_combine(d, norm_mode=L.MTP_NORM_ONE_PLUS_W)
    ref, _, flags = orc.combine(d["embed"], d["tokens"].numpy(), d["hidden"], d["w_norm_embed"],
                                d["w_norm_hidden"], d["eps"], d["fc"], norm_mode=1)
    plain, _, _ = orc.combine(d["embed"], d["tokens"].numpy(), d["hidden"], d["w_norm_embed"],
                              d["w_norm_hidden"], d["eps"], d["fc"], norm_mode=0)
    assert err == 0 and flags == 0
    assert_close(bf16_bits_to_f64(y), bf16_bits_to_f64(ref), "y")
    assert not np.allclose(bf16_bits_to_f64(plain), bf16_bits_to_f64(ref), rtol=0.05)


@pytest.mark.parametrize("h", [32, 512, 1024])
def test_combine_other_widths(orc, h):
    d = draft(3, seed=5, h=h, vocab=300)
    y, _ = gpu_combine(d)
    ref, _, _ = orc.combine(d["embed"], d["tokens"].numpy(), d["hidden"], d["w_norm_embed"],
                            d["w_norm_hidden"], d["eps"], d["fc"])
    assert_close(bf16_bits_to_f64(y), bf16_bits_to_f64(ref), "y")


def test_combine_bad_token_flag(orc):
    d = draft(2)
    toks = np.array([d["vocab"] + 5, 3], np.int32)
    y, err = gpu_combine(d, tokens=toks)
    assert err & L.MTP_DEVFLAG_BAD_TOKEN
    ref, _, flags = orc.combine(d["embed"], toks, d["hidden"], d["w_norm_embed"],
                                d["w_norm_hidden"], d["eps"], d["fc"])
    assert flags & 1
    assert_close(bf16_bits_to_f64(y), bf16_bits_to_f64(ref), "y")


@pytest.mark.parametrize("fmt", [1, 2])
def test_combine_quantized_fc(orc, fmt):
    d = draft(4, seed=6)
    h = d["h"]
    if fmt == 1:
        c, s = orc.quantize_fp8(d["fc"])
        fc = api.Table(1, h, 2 * h, to_dev(c), row_scale=to_dev(s))
        deq = orc.dequant(1, c, 2 * h, row_scale=s)
    else:
        c, b, g = orc.quantize_nvfp4(d["fc"])
        fc = api.Table(2, h, 2 * h, to_dev(c), block_scale=to_dev(pad_scales(b, 2 * h)),
                       global_scale=torch.tensor([g], dtype=torch.float32, device="cuda"))
        deq = orc.dequant(2, c, 2 * h, block_scale=b, global_scale=g)
    y, _ = gpu_combine(d, fc_table=fc)
    _, concat, _ = orc.combine(d["embed"], d["tokens"].numpy(), d["hidden"], d["w_norm_embed"],
                               d["w_norm_hidden"], d["eps"], d["fc"])
    ref = orc.f64_to_bf16(bf16_bits_to_f64(concat) @ deq.T)
    assert_close(bf16_bits_to_f64(y), bf16_bits_to_f64(ref), "y")


@pytest.mark.parametrize("M", [1, 4])
def test_tiny_draft_end_to_end(orc, M):
    """combine -> lm_head sweep -> argmax on the hidden-256 / vocab-4096 draft."""
    d = draft(M)
    y, _ = gpu_combine(d)
    head = api.LmHead(api.bf16_table(to_dev_u16(d["lm_head"])))
    idx, val, lg = head.argmax(to_dev_u16(y), logits=True)
    torch.cuda.synchronize()
    ref_y, _, _ = orc.combine(d["embed"], d["tokens"].numpy(), d["hidden"], d["w_norm_embed"],
                              d["w_norm_hidden"], d["eps"], d["fc"])
    ref_l, ref_i, ref_v, _ = orc.lm_head_argmax(0, d["lm_head"], d["h"], ref_y)
    for m in range(M):
        assert_argmax(int(idx[m].item()), ref_l[m])
        assert_close(bf16_bits_to_f64(u16_of(lg)[m]), ref_l[m], "logits")


def run_chain(dd, d, fc, head, steps, y_buf, idx_bufs, hid0):
    """Device-side draft chain: step j gathers the embedding of step j-1's argmax
    straight from the device index buffer (no host round trip); the combiner output
    stands in for the next hidden state (the drafter layer is not part of this path)."""
    tok = dd["tokens"]
    hid = hid0
    for j in range(steps):
        api.combine(dd["embed"], tok, hid, dd["w_norm_embed"], dd["w_norm_hidden"], d["eps"], fc,
                    out=y_buf[j])
        head(y_buf[j], idx_bufs[j])
        tok, hid = idx_bufs[j], y_buf[j]


@pytest.mark.parametrize("M", [1, 3])
def test_device_side_draft_chain(orc, M):
    """Four chained drafts on the device, eager and replayed from a CUDA graph (which
    admits no host synchronisation), against the oracle step by step."""
    steps = 4
    d = draft(M)
    dd = {k: (to_dev_u16(v) if isinstance(v, np.ndarray) and v.dtype == np.uint16 else v)
          for k, v in d.items()}
    dd["tokens"] = to_dev(np.asarray(d["tokens"], np.int32))
    fc = api.bf16_table(dd["fc"])
    head = api.LmHead(api.bf16_table(dd["lm_head"]))
    hid0 = dd["hidden"].clone()
    y_buf = [torch.empty((M, d["h"]), dtype=torch.bfloat16, device="cuda") for _ in range(steps)]
    idx_bufs = [torch.empty((M,), dtype=torch.int32, device="cuda") for _ in range(steps)]
    run_chain(dd, d, fc, head, steps, y_buf, idx_bufs, hid0)
    torch.cuda.synchronize()
    eager = [(u16_of(y).copy(), i.cpu().numpy().copy()) for y, i in zip(y_buf, idx_bufs)]
    # the oracle chain, continuing from the GPU's (valid) picks
    tok, hid = np.asarray(d["tokens"], np.int32), d["hidden"]
    for j in range(steps):
        ref_y, _, _ = orc.combine(d["embed"], tok, hid, d["w_norm_embed"], d["w_norm_hidden"],
                                  d["eps"], d["fc"])
        assert_close(bf16_bits_to_f64(eager[j][0]), bf16_bits_to_f64(ref_y), f"y step {j}")
        ref_l, _, _, _ = orc.lm_head_argmax(0, d["lm_head"], d["h"], eager[j][0])
        for m in range(M):
            assert_argmax(int(eager[j][1][m]), ref_l[m])
        tok, hid = eager[j][1], eager[j][0]
    # the same chain captured once and replayed: identical results
    for b in idx_bufs:
        b.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            run_chain(dd, d, fc, head, steps, y_buf, idx_bufs, hid0)
    g.replay()
    torch.cuda.synchronize()
    for j in range(steps):
        assert np.array_equal(u16_of(y_buf[j]), eager[j][0])
        assert np.array_equal(idx_bufs[j].cpu().numpy(), eager[j][1])


def gpu_draft_step(d, dd=None, mask=None, mask_words=0, stride=0, tokens=None, norm_mode=0):
    dd = dd or {k: (to_dev_u16(v) if isinstance(v, np.ndarray) and v.dtype == np.uint16 else v)
                for k, v in d.items()}
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    tok = to_dev(np.asarray(d["tokens"] if tokens is None else tokens, np.int32))
    m = to_dev(mask) if mask is not None else None
    idx, val, y = api.draft_step(dd["embed"], tok, dd["hidden"], dd["w_norm_embed"],
                                 dd["w_norm_hidden"], d["eps"], dd["fc"], dd["lm_head"], mask=m,
                                 mask_words=mask_words, mask_stride_words=stride, dev_err=err,
                                 norm_mode=norm_mode)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), val.cpu().numpy(), u16_of(y), int(err.item())


@pytest.mark.parametrize("M", [1, 2, 4])
def test_draft_step_one_launch(orc, M):
    """The fused draft step (one cluster launch): y and the argmax against the oracle."""
    d = draft(M)
    idx, val, y, err = gpu_draft_step(d)
    assert err == 0
    ref_y, _, _ = orc.combine(d["embed"], d["tokens"].numpy(), d["hidden"], d["w_norm_embed"],
                              d["w_norm_hidden"], d["eps"], d["fc"])
    assert_close(bf16_bits_to_f64(y), bf16_bits_to_f64(ref_y), "y")
    # the argmax over the GPU's own y (a bf16 ulp of y may move close logits)
    ref_l, _, _, _ = orc.lm_head_argmax(0, d["lm_head"], d["h"], y)
    for m in range(M):
        assert_argmax(int(idx[m]), ref_l[m])
        assert_close([val[m]], [ref_l[m].max()], "out_val")


@pytest.mark.parametrize("M", [1, 3])
def test_draft_step_one_plus_w(orc, M):
    d = draft(M, seed=78)
    idx, val, y, err = gpu_draft_step(d, norm_mode=L.MTP_NORM_ONE_PLUS_W)
    assert err == 0
    ref_y, _, _ = orc.combine(d["embed"], d["tokens"].numpy(), d["hidden"], d["w_norm_embed"],
                              d["w_norm_hidden"], d["eps"], d["fc"], norm_mode=1)
    assert_close(bf16_bits_to_f64(y), bf16_bits_to_f64(ref_y), "y")
    ref_l, _, _, _ = orc.lm_head_argmax(0, d["lm_head"], d["h"], y)
    for m in range(M):
        assert_argmax(int(idx[m]), ref_l[m])


# One input with h <= 256 and at most 256 head rows per CTA takes the register form (the
# weights held as MMA fragments); the rest, and every M > 1, the staged form (h 512:
# staged in shared memory; h 1024 with 5000 rows: read through L1). h 8 and 24 leave lanes
# without a k piece; 1000 rows leave a ragged last tile; 5000 rows at h 256 go staged.
@pytest.mark.parametrize("h,vocab,M", [(64, 1000, 1), (64, 1000, 2), (512, 3333, 1), (512, 3333, 2),
                                       (1024, 5000, 1), (1024, 5000, 2), (8, 300, 1), (24, 777, 1),
                                       (24, 777, 3), (256, 5000, 1), (256, 4000, 1)])
def test_draft_step_other_widths(orc, h, vocab, M):
    d = draft(M, seed=31 + h + vocab, h=h, vocab=vocab)
    idx, val, y, err = gpu_draft_step(d)
    assert err == 0
    ref_y, _, _ = orc.combine(d["embed"], d["tokens"].numpy(), d["hidden"], d["w_norm_embed"],
                              d["w_norm_hidden"], d["eps"], d["fc"])
    assert_close(bf16_bits_to_f64(y), bf16_bits_to_f64(ref_y), "y")
    ref_l, _, _, _ = orc.lm_head_argmax(0, d["lm_head"], d["h"], y)
    for m in range(M):
        assert_argmax(int(idx[m]), ref_l[m])
        assert_close([val[m]], [ref_l[m].max()], "out_val")


def test_draft_step_mask_and_flags(orc):
    """Per-input masks (one allowing nothing: index 0, -inf, the empty-mask flag) and a bad
    token id (a zero embedding row and the bad-token flag)."""
    d = draft(3)
    allowed, words = synth.keep_mask(17, 3, d["vocab"], 0.1)
    allowed[1] = False
    words[1] = 0
    W = words.shape[1]
    toks = np.asarray(d["tokens"], np.int32).copy()
    toks[2] = d["vocab"] + 5
    idx, val, y, err = gpu_draft_step(d, mask=words.reshape(-1), mask_words=W, stride=W, tokens=toks)
    assert err == (L.MTP_DEVFLAG_EMPTY_MASK | L.MTP_DEVFLAG_BAD_TOKEN)
    ref_y, _, _ = orc.combine(d["embed"], toks, d["hidden"], d["w_norm_embed"], d["w_norm_hidden"],
                              d["eps"], d["fc"])
    assert_close(bf16_bits_to_f64(y), bf16_bits_to_f64(ref_y), "y")
    ref_l, _, _, _ = orc.lm_head_argmax(0, d["lm_head"], d["h"], y)
    assert idx[1] == 0 and val[1] == -np.inf
    for m in (0, 2):
        assert_argmax(int(idx[m]), ref_l[m], allowed[m])


@pytest.mark.parametrize("keep", [0.1, 0.0])
def test_draft_step_mask_one_input(orc, keep):
    """One input (the register form) under a sparse mask, and under a mask allowing nothing
    (index 0, -inf, the empty-mask flag)."""
    d = draft(1, seed=91)
    allowed, words = synth.keep_mask(23, 1, d["vocab"], keep)
    W = words.shape[1]
    idx, val, y, err = gpu_draft_step(d, mask=words.reshape(-1), mask_words=W, stride=W)
    ref_l, _, _, _ = orc.lm_head_argmax(0, d["lm_head"], d["h"], y)
    if allowed[0].any():
        assert err == 0
        assert_argmax(int(idx[0]), ref_l[0], allowed[0])
    else:
        assert err == L.MTP_DEVFLAG_EMPTY_MASK
        assert idx[0] == 0 and val[0] == -np.inf


def test_draft_step_bad_token_one_input(orc):
    """One input (the register form) with a token id outside the vocabulary: a zero
    embedding row and the bad-token flag."""
    d = draft(1, seed=92)
    toks = np.asarray([d["vocab"] + 5], np.int32)
    idx, val, y, err = gpu_draft_step(d, tokens=toks)
    assert err == L.MTP_DEVFLAG_BAD_TOKEN
    ref_y, _, _ = orc.combine(d["embed"], toks, d["hidden"], d["w_norm_embed"], d["w_norm_hidden"],
                              d["eps"], d["fc"])
    assert_close(bf16_bits_to_f64(y), bf16_bits_to_f64(ref_y), "y")
    ref_l, _, _, _ = orc.lm_head_argmax(0, d["lm_head"], d["h"], y)
    assert_argmax(int(idx[0]), ref_l[0])


def test_draft_step_unaligned_norm_weights(orc):
    """Norm weights only 2-byte aligned (a view one element into a buffer): one input then
    takes the staged form, with the same results as the oracle."""
    d = draft(1, seed=93)
    dd = {k: (to_dev_u16(v) if isinstance(v, np.ndarray) and v.dtype == np.uint16 else v)
          for k, v in d.items()}
    for key in ("w_norm_embed", "w_norm_hidden"):
        buf = torch.empty((d["h"] + 1,), dtype=dd[key].dtype, device="cuda")
        buf[1:] = dd[key]
        dd[key] = buf[1:]
        assert dd[key].data_ptr() % 16 == 2
    idx, val, y, err = gpu_draft_step(d, dd=dd)
    assert err == 0
    ref_y, _, _ = orc.combine(d["embed"], d["tokens"].numpy(), d["hidden"], d["w_norm_embed"],
                              d["w_norm_hidden"], d["eps"], d["fc"])
    assert_close(bf16_bits_to_f64(y), bf16_bits_to_f64(ref_y), "y")
    ref_l, _, _, _ = orc.lm_head_argmax(0, d["lm_head"], d["h"], y)
    assert_argmax(int(idx[0]), ref_l[0])


def test_draft_step_chain_eager_and_graph(orc):
    """Eight chained fused steps (token and hidden from the previous step's outputs on the
    device), eager and replayed from a CUDA graph: identical, and each step matches the
    oracle from the previous step's GPU outputs."""
    steps, M = 8, 1
    d = draft(M)
    dd = {k: (to_dev_u16(v) if isinstance(v, np.ndarray) and v.dtype == np.uint16 else v)
          for k, v in d.items()}
    tok0 = to_dev(np.asarray(d["tokens"], np.int32))
    ys = [torch.empty((M, d["h"]), dtype=torch.bfloat16, device="cuda") for _ in range(steps)]
    ids = [torch.empty((M,), dtype=torch.int32, device="cuda") for _ in range(steps)]
    vals = [torch.empty((M,), dtype=torch.float32, device="cuda") for _ in range(steps)]

    def chain():
        tok, hid = tok0, dd["hidden"]
        for j in range(steps):
            api.draft_step(dd["embed"], tok, hid, dd["w_norm_embed"], dd["w_norm_hidden"], d["eps"],
                           dd["fc"], dd["lm_head"], out_y=ys[j], out_idx=ids[j], out_val=vals[j])
            tok, hid = ids[j], ys[j]

    chain()
    torch.cuda.synchronize()
    eager = [(u16_of(y).copy(), i.cpu().numpy().copy()) for y, i in zip(ys, ids)]
    tok, hid = np.asarray(d["tokens"], np.int32), d["hidden"]
    for j in range(steps):
        ref_y, _, _ = orc.combine(d["embed"], tok, hid, d["w_norm_embed"], d["w_norm_hidden"],
                                  d["eps"], d["fc"])
        assert_close(bf16_bits_to_f64(eager[j][0]), bf16_bits_to_f64(ref_y), f"y step {j}")
        ref_l, _, _, _ = orc.lm_head_argmax(0, d["lm_head"], d["h"], eager[j][0])
        assert_argmax(int(eager[j][1][0]), ref_l[0])
        tok, hid = eager[j][1], eager[j][0]
    for b in ids:
        b.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            chain()
    g.replay()
    torch.cuda.synchronize()
    for j in range(steps):
        assert np.array_equal(u16_of(ys[j]), eager[j][0])
        assert np.array_equal(ids[j].cpu().numpy(), eager[j][1])
