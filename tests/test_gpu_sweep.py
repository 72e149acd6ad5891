"""The fused lm_head sweep + argmax on the GPU against the oracle.

Small tables span several 16-row tiles, several CTAs and a ragged tail; the full
tables are the benchmark's (154,880 x 4,096 BF16 and FP8, 131,072 x 5,120 NVFP4) in
the launch configuration bench.py times. Logits within 2e-2 + 1e-2|ref|; argmax exact
where the top-2 gap exceeds 1e-2; one-hot inputs and batch invariance bit-exact within
each range of M that one sweep serves (BF16 1-8, 9-16, 17-32; FP8 1-6, 7-16, 17-32; NVFP4
1-2, 3-16, 17-32)."""
import numpy as np
import pytest
import torch

from helpers import (allowed_from_mask, assert_argmax, assert_close, bf16_bits_to_f64,
                     pad_scales, to_dev, to_dev_u16, u16_of)
from mtp_speculative_draft_lm_b200 import _lib as L
from mtp_speculative_draft_lm_b200 import api, synth

pytestmark = pytest.mark.gpu


def oracle_quant(orc, w_u16, fmt):
    if fmt == 0:
        return dict(data=w_u16)
    if fmt == 1:
        c, s = orc.quantize_fp8(w_u16)
        return dict(data=c, row_scale=s)
    c, b, g = orc.quantize_nvfp4(w_u16)
    return dict(data=c, block_scale=b, global_scale=g)


def device_table(q, fmt, n, k):
    if fmt == 0:
        return api.Table(0, n, k, to_dev_u16(q["data"]))
    if fmt == 1:
        return api.Table(1, n, k, to_dev(q["data"]), row_scale=to_dev(q["row_scale"]))
    return api.Table(2, n, k, to_dev(q["data"]), block_scale=to_dev(pad_scales(q["block_scale"], k)),
                     global_scale=torch.tensor([q["global_scale"]], dtype=torch.float32,
                                               device="cuda"))


def run_sweep(table, x_u16, n_eff=None, mask=None, mask_words=0, stride=0, logits=True,
              head=None):
    head = head or api.LmHead(table, n_eff)
    x = to_dev_u16(x_u16)
    m = to_dev(mask) if mask is not None else None
    head.dev_err.zero_()
    idx, val, lg = head.argmax(x, mask=m, mask_words=mask_words, mask_stride_words=stride,
                               logits=logits)
    torch.cuda.synchronize()
    return (idx.cpu().numpy(), val.cpu().numpy(), u16_of(lg) if logits else None,
            int(head.dev_err.item()))


def oracle_sweep(orc, q, fmt, k, x_u16, n_eff=None, mask=None, mask_words=0, stride=0):
    return orc.lm_head_argmax(fmt, q["data"], k, x_u16, n_eff=n_eff,
                              row_scale=q.get("row_scale"), block_scale=q.get("block_scale"),
                              global_scale=q.get("global_scale", 0.0), mask=mask,
                              mask_words=mask_words, mask_stride_words=stride)


def check(orc, fmt, q, k, x_u16, got, n_eff=None, mask=None, mask_words=0, stride=0):
    idx, val, lg, flags = got
    ref_l, ref_i, ref_v, ref_f = oracle_sweep(orc, q, fmt, k, x_u16, n_eff, mask, mask_words,
                                              stride)
    M, n = ref_l.shape
    for m in range(M):
        allowed = None
        if mask is not None:
            allowed = allowed_from_mask(mask[m * stride: m * stride + mask_words] if stride
                                        else mask[:mask_words], n, mask_words)
        if allowed is not None and not allowed.any():
            assert idx[m] == 0 and val[m] == -np.inf
            continue
        assert_argmax(int(idx[m]), ref_l[m], allowed)
        assert_close([val[m]], [ref_v[m]], "out_val")
        if lg is not None:
            gl = bf16_bits_to_f64(lg[m])
            if allowed is not None:
                assert np.all(np.isneginf(gl[~allowed]))
                assert_close(gl[allowed], ref_l[m][allowed], f"logits row {m}")
            else:
                assert_close(gl, ref_l[m], f"logits row {m}")
    assert (flags & L.MTP_DEVFLAG_EMPTY_MASK) == (ref_f & 2)


SHAPES = {0: [(1000, 256), (1000, 4096), (4133, 576)],
          1: [(1000, 128), (1000, 4096), (517, 1152)],
          2: [(1000, 256), (1000, 5120), (517, 1280)]}


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("M", [1, 3, 6, 7, 8, 9, 16, 17, 32])
def test_sweep_small_tables(orc, fmt, M):
    for n, k in SHAPES[fmt]:
        w = synth.as_u16(synth.normal_bf16(synth._gen(n + k + fmt), (n, k), 0.02))
        x = synth.as_u16(synth.normal_bf16(synth._gen(7 + M), (M, k), 1.0))
        q = oracle_quant(orc, w, fmt)
        got = run_sweep(device_table(q, fmt, n, k), x)
        check(orc, fmt, q, k, x, got)


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_one_hot_inputs_are_bit_exact(orc, fmt):
    n, k = 777, 256
    w = synth.as_u16(synth.normal_bf16(synth._gen(5), (n, k), 0.02))
    q = oracle_quant(orc, w, fmt)
    table = device_table(q, fmt, n, k)
    for j in (0, 77, k - 1):
        x = np.zeros((1, k), np.float32)
        x[0, j] = 1.0
        xu = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        idx, val, lg, _ = run_sweep(table, xu)
        ref_l, ref_i, ref_v, _ = oracle_sweep(orc, q, fmt, k, xu)
        assert np.float32(ref_v[0]) == val[0]  # the winning entry, exactly
        assert idx[0] == ref_i[0]              # ties resolved to the lowest row alike
        want = orc.f64_to_bf16(ref_l[0].astype(np.float32).astype(np.float64))
        assert np.array_equal(lg[0], want)


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_batch_invariance(orc, fmt):
    n, k = 2000, 1024
    w = synth.as_u16(synth.normal_bf16(synth._gen(9), (n, k), 0.02))
    x = synth.as_u16(synth.normal_bf16(synth._gen(10), (32, k), 1.0))
    table = device_table(oracle_quant(orc, w, fmt), fmt, n, k)
    head = api.LmHead(table)
    # Several sweeps share the work: NVFP4 with one or two inputs applies the block scales
    # to per-block fp32 sums, 3-16 inputs run on block-scaled FP4 MMAs (each accumulator
    # column computed alike whatever the MMA's width), 17-32 on the tensor-memory sweep;
    # more inputs (BF16 from 9, FP8 from 7) go to the tcgen05 sweep with 16 or 32 MMA
    # columns. Each sums its products in its own fixed order, so results are bit-identical
    # within each range of M and within the tolerance across them
    groups = {0: [(1, 2, 3, 4, 8), (9, 12, 16), (17, 24, 32)],
              1: [(1, 2, 3, 4, 6), (7, 8, 12, 16), (17, 24, 32)],
              2: [(1, 2), (3, 4, 8, 9, 12, 16), (17, 24, 32)]}[fmt]
    bases = []
    for grp in groups:
        base = run_sweep(table, x[:grp[0]], head=head)
        bases.append(base)
        for M in grp[1:]:
            got = run_sweep(table, x[:M], head=head)
            assert np.array_equal(got[2][0], base[2][0]), M
            assert got[1][0].view(np.uint32) == base[1][0].view(np.uint32)
    for b in bases[1:]:
        assert_close(bf16_bits_to_f64(b[2][0]), bf16_bits_to_f64(bases[0][2][0]), "across ranges of M")
    # row m keeps its result whatever the other rows are
    x2 = x.copy()
    x2[1:] = x[::-1][:31]
    for M in (2, 16, 32):
        a = run_sweep(table, x[:M], head=head)
        b = run_sweep(table, x2[:M], head=head)
        assert np.array_equal(a[2][0], b[2][0]), M


def test_masks_decoys_and_edge_cases(orc):
    n, k, M = 5000, 512, 4
    d = synth.head_table(11, n, k, M, mask_keep=0.1)
    w, x = synth.as_u16(d["W"]), synth.as_u16(d["x"])
    for fmt in (0, 1, 2):
        q = oracle_quant(orc, w, fmt)
        table = device_table(q, fmt, n, k)
        words = d["mask"].shape[1]
        got = run_sweep(table, x)
        assert np.array_equal(got[0], d["top"])
        mask = d["mask"].reshape(-1)
        got = run_sweep(table, x, mask=mask, mask_words=words, stride=words)
        assert np.array_equal(got[0], d["second"])
        check(orc, fmt, q, k, x, got, mask=mask, mask_words=words, stride=words)
        # one shared mask (stride 0)
        got = run_sweep(table, x, mask=d["mask"][1], mask_words=words, stride=0)
        check(orc, fmt, q, k, x, got, mask=d["mask"][1], mask_words=words, stride=0)
        # a mask shorter than the vocab disallows everything past it
        got = run_sweep(table, x, mask=mask, mask_words=3, stride=words)
        check(orc, fmt, q, k, x, got, mask=mask, mask_words=3, stride=words)
    # an all-zero mask row: index 0, -inf, and the empty-mask flag
    q = oracle_quant(orc, w, 0)
    table = device_table(q, 0, n, k)
    mask = d["mask"].copy()
    mask[2] = 0
    got = run_sweep(table, x, mask=mask.reshape(-1), mask_words=mask.shape[1],
                    stride=mask.shape[1])
    assert got[0][2] == 0 and got[1][2] == -np.inf
    assert got[3] & L.MTP_DEVFLAG_EMPTY_MASK
    assert L.mtp_devflags_status(got[3]) == L.MTP_WARN_EMPTY_MASK
    assert np.array_equal(got[0][[0, 1, 3]], d["second"][[0, 1, 3]])


@pytest.mark.parametrize("M", [7, 12, 32])
def test_masks_and_n_eff_many_inputs(orc, M):
    """The sweeps that stream x per K chunk (tcgen05 for BF16 / FP8, 64-row tiles for
    NVFP4): per-row masks with a decoy, a shared mask, an all-zero mask row, masked logits
    -inf, and an n_eff that ends mid-tile."""
    n, k = 4133, 512
    d = synth.head_table(13 + M, n, k, M, mask_keep=0.1)
    w, x = synth.as_u16(d["W"]), synth.as_u16(d["x"])
    words = d["mask"].shape[1]
    for fmt in (0, 1, 2):
        q = oracle_quant(orc, w, fmt)
        table = device_table(q, fmt, n, k)
        got = run_sweep(table, x)
        assert np.array_equal(got[0], d["top"])
        mask = d["mask"].copy()
        mask[M // 2] = 0
        got = run_sweep(table, x, mask=mask.reshape(-1), mask_words=words, stride=words)
        check(orc, fmt, q, k, x, got, mask=mask.reshape(-1), mask_words=words, stride=words)
        keep = [m for m in range(M) if m != M // 2]
        assert np.array_equal(got[0][keep], d["second"][keep])
        assert got[0][M // 2] == 0 and got[1][M // 2] == -np.inf
        got = run_sweep(table, x, mask=d["mask"][0], mask_words=words, stride=0)
        check(orc, fmt, q, k, x, got, mask=d["mask"][0], mask_words=words, stride=0)
        got = run_sweep(table, x, n_eff=2011)
        check(orc, fmt, q, k, x, got, n_eff=2011)


def test_duplicate_rows_lowest_index_and_n_eff(orc):
    n, k = 3000, 256
    d = synth.head_table(12, n, k, 1)
    w = synth.as_u16(d["W"]).copy()
    top = int(d["top"][0])
    dups = sorted({5, 1500, 2999, top})
    for r in dups:
        w[r] = w[top]
    table = device_table(dict(data=w), 0, n, k)
    got = run_sweep(table, synth.as_u16(d["x"]))
    assert got[0][0] == dups[0]
    got = run_sweep(table, synth.as_u16(d["x"]), n_eff=1234)
    check(orc, 0, dict(data=w), k, synth.as_u16(d["x"]), got, n_eff=1234)
    assert got[2].shape == (1, 1234)


def test_workspace_reuse_across_calls(orc):
    n, k = 4000, 256
    d = synth.head_table(13, n, k, 2)
    table = device_table(dict(data=synth.as_u16(d["W"])), 0, n, k)
    head = api.LmHead(table)
    for _ in range(5):
        got = run_sweep(table, synth.as_u16(d["x"]), head=head)
        assert np.array_equal(got[0], d["top"])
        assert int(head.ws[:4].view(torch.int32).item()) == 0


FULL = [(synth.BF16_HEAD, 0), (synth.FP8_HEAD, 1), (synth.NVFP4_HEAD, 2)]


@pytest.mark.parametrize("cfg,fmt", FULL, ids=["bf16", "fp8", "nvfp4"])
def test_full_tables(orc, cfg, fmt):
    Mmax = max(cfg["Ms"])
    d = synth.head_table(cfg["seed"], cfg["N"], cfg["K"], Mmax,
                         mask_keep=cfg.get("mask_keep"))
    w, x = synth.as_u16(d["W"]), synth.as_u16(d["x"])
    q = oracle_quant(orc, w, fmt)
    table = device_table(q, fmt, cfg["N"], cfg["K"])
    head = api.LmHead(table)
    ref_l, ref_i, ref_v, _ = oracle_sweep(orc, q, fmt, cfg["K"], x)
    for M in cfg["Ms"]:
        idx, val, lg, _ = run_sweep(table, x[:M], head=head)
        assert np.array_equal(idx, d["top"][:M])
        assert np.array_equal(idx, ref_i[:M])
        assert_close(val, ref_v[:M], "out_val")
        rows = np.random.default_rng(M).choice(cfg["N"], 20000, replace=False)
        assert_close(bf16_bits_to_f64(lg[:, rows]), ref_l[:M, rows], "logits sample")
    if "mask" in d:
        words = d["mask"].shape[1]
        for M in cfg["Ms"]:
            got = run_sweep(table, x[:M], head=head, mask=d["mask"][:M].reshape(-1),
                            mask_words=words, stride=words, logits=False)
            assert np.array_equal(got[0], d["second"][:M])


# Inputs for which the masked sweep (which reads only allowed rows) and the unmasked one
# run the same kernel, so that their logits must agree bit for bit (NVFP4: none, the
# unmasked sweep runs on block-scaled FP4 MMAs, the gathered one on decoded f16 MMAs).
SAME_KERNEL_M = {0: 8, 1: 6, 2: 0}


@pytest.mark.parametrize("cfg,fmt", FULL, ids=["bf16", "fp8", "nvfp4"])
def test_masked_full_tables(orc, cfg, fmt):
    """Grammar masks keeping 1% and 50% of the tokens on the full tables (the masked sweep
    reads only the rows some input allows): the masked argmax and value against the oracle,
    every disallowed logit -inf, every allowed logit within tolerance of the oracle on a
    sample, and identical to the unmasked sweep's where both run the same kernel."""
    Ms = (1, 4, 8) if fmt != 2 else (1, 2, 4)
    Mmax = max(Ms)
    N, K = cfg["N"], cfg["K"]
    d = synth.head_table(cfg["seed"], N, K, Mmax)
    w, x = synth.as_u16(d["W"]), synth.as_u16(d["x"])
    q = oracle_quant(orc, w, fmt)
    table = device_table(q, fmt, N, K)
    head = api.LmHead(table)
    ref_l, _, _, _ = oracle_sweep(orc, q, fmt, K, x)
    dense = {M: run_sweep(table, x[:M], head=head)[2] for M in Ms if M <= SAME_KERNEL_M[fmt]}
    sample = np.random.default_rng(fmt).choice(N, 5000, replace=False)
    for keep in (0.01, 0.5):
        allowed, words = synth.keep_mask(int(keep * 1000) + fmt, Mmax, N, keep)
        W = words.shape[1]
        for M in Ms:
            idx, val, lg, flags = run_sweep(table, x[:M], head=head, mask=words[:M].reshape(-1),
                                            mask_words=W, stride=W)
            assert flags == 0
            for m in range(M):
                a = allowed[m]
                assert_argmax(int(idx[m]), ref_l[m], a)
                assert_close([val[m]], [ref_l[m][a].max()], "masked out_val")
                assert np.all(lg[m][~a] == 0xFF80)
                rs = sample[a[sample]]
                assert_close(bf16_bits_to_f64(lg[m][rs]), ref_l[m][rs], "masked logits sample")
                if M in dense:
                    assert np.array_equal(lg[m][a], dense[M][m][a]), (keep, M, m)
        # one mask shared by every input (stride 0)
        idx, val, lg, _ = run_sweep(table, x[:2], head=head, mask=words[0], mask_words=W, stride=0)
        for m in range(2):
            assert_argmax(int(idx[m]), ref_l[m], allowed[0])
            if 2 <= SAME_KERNEL_M[fmt]:
                two = run_sweep(table, x[:2], head=head)[2]
                assert np.array_equal(lg[m][allowed[0]], two[m][allowed[0]])


def oracle_logprobs(orc, ref_l, mask=None, mask_words=0, stride=0):
    out = []
    for m in range(ref_l.shape[0]):
        mrow = None
        if mask is not None:
            mrow = mask[m * stride: m * stride + mask_words] if stride else mask[:mask_words]
        out.append(orc.top1_logprob(ref_l[m], mrow, mask_words))
    return np.array(out)


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("M", [1, 2, 3, 9, 16, 32])
def test_top1_logprob(orc, fmt, M):
    """mtp_lm_head_argmax_lp: the argmax outputs equal mtp_lm_head_argmax's bit for bit,
    and the top-1 log-probability matches the oracle's (fp64 log-softmax at the argmax)
    within 2e-2 + 1e-2|ref|, with and without a mask; an all-masked row gives -inf."""
    n, k = 3000, {0: 512, 1: 1024, 2: 1280}[fmt]
    w = synth.as_u16(synth.normal_bf16(synth._gen(40 + fmt), (n, k), 0.05))
    x = synth.as_u16(synth.normal_bf16(synth._gen(50 + M), (M, k), 1.0))
    q = oracle_quant(orc, w, fmt)
    table = device_table(q, fmt, n, k)
    head = api.LmHead(table)
    xd = to_dev_u16(x)
    i0, v0, l0 = head.argmax(xd, logits=True)
    i1, v1, l1, lp = head.argmax(xd, logits=True, logprob=True)
    torch.cuda.synchronize()
    assert torch.equal(i0, i1) and torch.equal(v0.view(torch.int32), v1.view(torch.int32))
    assert torch.equal(l0.view(torch.int16), l1.view(torch.int16))
    ref_l, ref_i, _, _ = oracle_sweep(orc, q, fmt, k, x)
    assert np.array_equal(i1.cpu().numpy(), ref_i)
    assert_close(lp.cpu().numpy(), oracle_logprobs(orc, ref_l), "top-1 log-probability")
    assert np.all(lp.cpu().numpy() <= 0.0)
    # per-row masks keeping ~5%; row 0 keeps nothing
    words = (n + 31) // 32
    rng = np.random.default_rng(60 + M)
    keep = rng.random((M, words * 32)) < 0.05
    keep[0] = False
    bits = keep.reshape(M, words, 32).astype(np.uint64) << np.arange(32, dtype=np.uint64)
    mask = bits.sum(axis=-1).astype(np.uint32).view(np.int32)
    md = to_dev(mask.reshape(-1))
    _, _, _, lpm = head.argmax(xd, mask=md, mask_words=words, mask_stride_words=words,
                               logprob=True)
    torch.cuda.synchronize()
    got = lpm.cpu().numpy()
    ref = oracle_logprobs(orc, ref_l, mask.reshape(-1), words, words)
    assert got[0] == -np.inf and ref[0] == -np.inf
    assert_close(got[1:], ref[1:], "masked top-1 log-probability")


@pytest.mark.parametrize("cfg,fmt", FULL, ids=["bf16", "fp8", "nvfp4"])
def test_top1_logprob_full_tables(orc, cfg, fmt):
    d = synth.head_table(cfg["seed"], cfg["N"], cfg["K"], 1)
    w, x = synth.as_u16(d["W"]), synth.as_u16(d["x"])
    q = oracle_quant(orc, w, fmt)
    table = device_table(q, fmt, cfg["N"], cfg["K"])
    head = api.LmHead(table)
    idx, _, _, lp = head.argmax(to_dev_u16(x), logprob=True)
    torch.cuda.synchronize()
    ref_l, ref_i, _, _ = oracle_sweep(orc, q, fmt, cfg["K"], x)
    assert idx.item() == ref_i[0]
    assert_close(lp.cpu().numpy(), oracle_logprobs(orc, ref_l), "full-table log-probability")


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("M", [1, 3, 12])
def test_host_input_and_result(orc, fmt, M):
    """mtp_lm_head_argmax_host: x read from pinned host memory and (index, value) written
    to pinned host memory by the call itself; several calls in a row on one stream, each
    with new input bytes, match the device-buffer entry point."""
    n, k = 1500, 512
    d = synth.head_table(21 + M, n, k, M)
    q = oracle_quant(orc, synth.as_u16(d["W"]), fmt)
    table = device_table(q, fmt, n, k)
    head = api.LmHead(table)
    out = torch.empty((3, 2 * M), dtype=torch.int32).pin_memory()
    xs = []
    for j in range(3):
        x = d["x"] if j == 0 else synth.normal_bf16(synth._gen(50 + j), (M, k), 1.0)
        xh = x.contiguous().pin_memory()
        xs.append(xh)
        head.argmax_host(xh, out[j])  # three steps queued back to back
    torch.cuda.synchronize()
    assert np.array_equal(out[0, :M].numpy(), d["top"])
    for j in range(3):
        idx, val, _ = head.argmax(xs[j].cuda())
        torch.cuda.synchronize()
        assert np.array_equal(out[j, :M].numpy(), idx.cpu().numpy())
        assert np.array_equal(out[j, M:].numpy(), val.cpu().view(torch.int32).numpy())
    # pageable host memory is refused
    with pytest.raises(L.MtpError):
        head.argmax_host(d["x"].contiguous(), out[0])
